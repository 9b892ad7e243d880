// layout_dispatch.cu -- the dispatch layout and the dispatch of the same
// batch in ONE launch, for small batches such as a decode step.
//
// DeepEP keeps separate low-latency kernels for small decode batches
// (dataforcee.us rewrite, "Technological Views and Benefits": 128 tokens,
// eight experts).  Inside one GPU such a step is bound by launch and
// dependency latency, not by bytes, so this path drops the layout launch
// and the wait between it and the dispatch: every CTA works out the
// layout entries it needs from the ids themselves (a few KB, served by L2
// after the first CTA reads them), with no CTA ever waiting on another,
// then dispatches its own tokens and writes their layout entries.  The
// token rows are bulk-loaded (cp.async.bulk) as the kernel starts, and the
// FP8 cast, which does not need the layout, runs while the layout work is
// in flight.  Results are bit-identical to ep_get_layout followed by
// ep_dispatch.
//
// Two kernels:
//  * layout_dispatch_token_kernel (T + 1 CTAs fit on the GPU at once, e.g.
//    a 128-token decode step): CTA b < T owns token b only.  The receive
//    row of its slot (b, j) with expert e is the number of kept slots whose
//    (expert, flat slot index) key is smaller than (e, b*k + j): expert-
//    major, token-major inside an expert -- the stable order of the unfused
//    layout, duplicates included.  The CTA counts those keys over all ids
//    (each thread a strided share, a warp-wide sum per slot, then the
//    warps' sums added by one thread per slot), so it needs no table, no
//    scan and no zeroing; it casts
//    its row while the ids are in flight.  CTA T alone builds the
//    per-expert and per-rank counts and offsets.
//  * layout_dispatch_kernel (larger batches): CTAs own contiguous token
//    ranges.  Warps 0..7 of every CTA build the whole layout in shared
//    memory as one token bit set per expert (bit t % 32 of mask[e][t / 32]
//    set when token t chose expert e), per-expert counts and their scan;
//    meanwhile warps 8..23 cast the CTA's first row.  The receive row of
//    slot (t, j) with expert e is off_e[e] + (tokens before t that chose
//    e), a popcount of the set below bit t.  A token naming one expert
//    twice (two slots, as the unfused path accepts) is seen while the sets
//    are built; the ranks are then counted over the flat slot order
//    instead.  CTA 0 writes the counts and offsets; k threads issue each
//    token's bulk stores, one receive row each.
#include <cuda_bf16.h>

#include "bulk.cuh"
#include "ep_internal.cuh"
#include "fp8.cuh"

namespace ep {
namespace {

constexpr int kLayoutThreads = 256;  // warps 0..7: the layout
constexpr int kLayoutWarps = kLayoutThreads / kWarp;
constexpr int kCastThreads = 512;    // warps 8..23: the first row's FP8 cast
constexpr int kThreads = kLayoutThreads + kCastThreads;
constexpr int kStages = 2;             // token rows in flight per CTA
constexpr long kMaxSlots = 8192;       // T * k of the fused path
constexpr long kMaxMaskBytes = 32768;  // E * ceil(T / 32) * 4
constexpr int kMaxH = 16384;
constexpr int kLayoutBarrier = 1;      // named barrier of the layout warps

__host__ __device__ constexpr int align16(long b) { return static_cast<int>((b + 15) & ~15L); }

// Byte offsets of the dynamic shared memory regions (host and device agree).
struct SmemMap {
  int in, out_q, out_s, mask, cnt, off, cnt_r, ids, rows, total;
};

__host__ __device__ inline SmemMap smem_map(int T, int k, int E, int R, int H, bool fp8,
                                            int per_cta) {
  SmemMap m;
  const long W = (T + 31) / 32;
  int o = 0;
  m.in = o;     o += kStages * 2 * H;           // bf16 rows: 2H is a multiple of 16
  m.out_q = o;  o += fp8 ? H : 0;               // e4m3 row
  m.out_s = o;  o += fp8 ? H / 32 : 0;          // H / 128 fp32 scales
  m.mask = o;   o += align16(E * W * 4);
  m.cnt = o;    o += align16(static_cast<long>(E) * 4);
  m.off = o;    o += align16(static_cast<long>(E + 1) * 4);
  m.cnt_r = o;  o += align16(static_cast<long>(R) * 4);
  m.ids = o;    o += align16(static_cast<long>(T) * k * 2);
  m.rows = o;   o += align16(static_cast<long>(per_cta) * k * 4);  // this CTA's receive rows
  m.total = o;
  return m;
}

struct FusedArgs {
  const void *idx;
  int T, k, E, R, G, H, W;
  unsigned long long g_magic;  // ceil(2^32 / G): e / G == (e * g_magic) >> 32 for e < 1024
  const uint4 *x;
  int32_t *cnt_e, *cnt_r, *off_e, *off_r, *slot_pos, *recv_src;
  uint8_t *in_rank;
  unsigned char *recv;  // bf16 [T*k, H] or e4m3 [T*k, H]
  float *recv_scale;    // [T*k, H / 128] (FP8)
  int32_t *d_err;
  int per_cta;          // tokens per CTA
  int first_polls;      // poll limit of each CTA's first row wait
};

__device__ __forceinline__ void layout_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kLayoutBarrier), "n"(kLayoutThreads) : "memory");
}

__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

__device__ __forceinline__ int warp_sum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// out[0..n) = exclusive scan of in[0..n), out[n] = total, by the layout
// warps (each thread a contiguous run of ceil(n / kLayoutThreads) entries).
__device__ void layout_exclusive_scan(const int *in, int *out, int n, int *warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kLayoutThreads - 1) / kLayoutThreads;
  const int b = min(n, tid * per), e = min(n, b + per);
  int local = 0;
  for (int q = b; q < e; ++q) local += in[q];
  const int incl = warp_incl_scan(local);
  if (lane == 31) warp_tot[warp] = incl;
  layout_sync();
  if (warp == 0) {
    const int v = lane < kLayoutWarps ? warp_tot[lane] : 0;
    const int iv = warp_incl_scan(v);
    if (lane < kLayoutWarps) warp_tot[lane] = iv - v;
    if (lane == kLayoutWarps - 1) out[n] = iv;
  }
  layout_sync();
  int run = warp_tot[warp] + incl - local;
  for (int q = b; q < e; ++q) {
    out[q] = run;
    run += in[q];
  }
}

// e4m3 codes and scales of one bf16 row (smem) into the output stage, by
// the `nthreads` threads numbered ctid = 0..nthreads-1 (a multiple of 32):
// a half-warp per 128-channel block; whole warps share the loop bound
// because H / 8 is a multiple of 64.
__device__ __forceinline__ void cast_row(const uint4 *xin, uint2 *qo, float *so, int H, int ctid,
                                         int nthreads) {
  for (int v = ctid; v < (H >> 3); v += nthreads) {
    float sc;
    qo[v] = quantize_block_lane(xin[v], &sc);
    if ((ctid & 15) == 0) so[v >> 4] = sc;
  }
}

template <typename IdT, bool kFp8>
__global__ void __launch_bounds__(kThreads) layout_dispatch_kernel(const FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const SmemMap sm = smem_map(a.T, a.k, a.E, a.R, a.H, kFp8, a.per_cta);
  unsigned char *in_buf = smem + sm.in;
  uint2 *out_q = reinterpret_cast<uint2 *>(smem + sm.out_q);
  float *out_s = reinterpret_cast<float *>(smem + sm.out_s);
  unsigned *mask = reinterpret_cast<unsigned *>(smem + sm.mask);
  int *cnt = reinterpret_cast<int *>(smem + sm.cnt);
  int *off = reinterpret_cast<int *>(smem + sm.off);
  int *cnt_r = reinterpret_cast<int *>(smem + sm.cnt_r);
  int16_t *ids = reinterpret_cast<int16_t *>(smem + sm.ids);
  int *rows = reinterpret_cast<int *>(smem + sm.rows);  // [per_cta][k]
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int warp_tot[kLayoutWarps];
  __shared__ int dup;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, k = a.k, E = a.E, R = a.R, G = a.G, H = a.H, W = a.W;
  const int N = T * k;
  const int first = blockIdx.x * a.per_cta;
  const int n_mine = max(0, min(T, first + a.per_cta) - first);
  const int in_bytes = 2 * H;
  const bool lead = blockIdx.x == 0;

  // thread 0: token first + i -> input stage i % kStages
  auto issue = [&](int i) {
    const int s = i % kStages;
    mbar_arrive_expect_tx(&full[s], in_bytes);
    bulk_load(in_buf + s * in_bytes, a.x + static_cast<long>(first + i) * (H >> 3), in_bytes,
              &full[s]);
  };
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
    dup = 0;
    pdl_wait();  // rows and ids come from the previous kernel on the stream
    for (int i = 0; i < min(kStages, n_mine); ++i) issue(i);
  }
  for (int q = tid; q < E * W; q += kThreads) mask[q] = 0u;
  for (int q = tid; q < E; q += kThreads) cnt[q] = 0;
  for (int q = tid; q < R; q += kThreads) cnt_r[q] = 0;
  pdl_wait();
  __syncthreads();

  bool ok = true;  // this thread's row wait did not time out
  if (tid < kLayoutThreads) {
    // ---- the layout (warps 0..7) ----
    // 1. ids -> per-expert token sets and slot counts (bad ids reported once)
    const IdT *idx = static_cast<const IdT *>(a.idx);
    constexpr int kBatch = 4;
    for (int base = 0; base < N; base += kBatch * kLayoutThreads) {
      long long v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kLayoutThreads + tid;
        v[u] = i < N ? static_cast<long long>(idx[i]) : -1;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = base + u * kLayoutThreads + tid;
        if (i >= N) continue;
        int e = -1;
        if (v[u] >= 0 && v[u] < E)
          e = static_cast<int>(v[u]);
        else if (v[u] != -1 && lead && a.d_err != nullptr)
          atomicExch(reinterpret_cast<int *>(a.d_err), EP_ERR_INDEX);
        ids[i] = static_cast<int16_t>(e);
        if (e >= 0) {
          const int t = i / k;
          const unsigned bit = 1u << (t & 31);
          if (atomicOr(&mask[e * W + (t >> 5)], bit) & bit) dup = 1;
          atomicAdd(&cnt[e], 1);
        }
      }
    }
    layout_sync();

    // 2. offsets; CTA 0 also counts the tokens of each rank (a token's ranks
    //    as a bit mask over its ids, R <= 64)
    if (lead) {
      for (int t = tid; t < T; t += kLayoutThreads) {
        unsigned long long rm = 0ull;
        for (int j = 0; j < k; ++j) {
          const int e = ids[t * k + j];
          if (e >= 0) rm |= 1ull << ((static_cast<unsigned long long>(e) * a.g_magic) >> 32);
        }
        while (rm != 0ull) {
          atomicAdd(&cnt_r[__ffsll(static_cast<long long>(rm)) - 1], 1);
          rm &= rm - 1ull;
        }
      }
    }
    layout_exclusive_scan(cnt, off, E, warp_tot);
    layout_sync();
    const int n_eff = off[E];
    if (lead) {
      for (int q = tid; q < E; q += kLayoutThreads) {
        a.cnt_e[q] = cnt[q];
        a.off_e[q] = off[q];
      }
      if (tid == 0) a.off_e[E] = n_eff;
      if (warp == kLayoutWarps - 1) {
        int carry = 0;
        for (int b = 0; b < R; b += 32) {
          const int r = b + lane;
          const int c = r < R ? cnt_r[r] : 0;
          const int incl = warp_incl_scan(c);
          if (r < R) {
            a.cnt_r[r] = c;
            a.off_r[r] = carry + incl - c;
          }
          carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) a.off_r[R] = carry;
      }
    }
    // receive rows no slot points at
    for (int r = n_eff + blockIdx.x * kLayoutThreads + tid; r < N;
         r += gridDim.x * kLayoutThreads)
      a.recv_src[r] = -1;

    // 3. receive rows of this CTA's slots: a thread per slot when the token
    //    sets are short (<= 4 words), else a warp per slot
    const int n_slots = n_mine * k;
    const int f0 = first * k;
    auto place = [&](int q, int before) {
      const int e = ids[f0 + q];
      const int row = e >= 0 ? off[e] + before : -1;
      rows[q] = row;
      a.slot_pos[f0 + q] = row;
      if (row >= 0) a.recv_src[row] = first + q / k;
    };
    if (!dup && W <= 4) {
      for (int q = tid; q < n_slots; q += kLayoutThreads) {
        const int e = ids[f0 + q];
        int c = 0;
        if (e >= 0) {
          const int t = first + q / k;
          const unsigned *me = mask + e * W;
          for (int w = 0; w < (t >> 5); ++w) c += __popc(me[w]);
          c += __popc(me[t >> 5] & ((1u << (t & 31)) - 1u));
        }
        place(q, c);
      }
    } else {
      for (int q = warp; q < n_slots; q += kLayoutWarps) {
        const int e = ids[f0 + q];
        int c = 0;
        if (e >= 0) {
          if (!dup) {  // tokens before t that chose e
            const int t = first + q / k;
            const unsigned *me = mask + e * W;
            const int wt = t >> 5;
            for (int w = lane; w < wt; w += 32) c += __popc(me[w]);
            if (lane == 0) c += __popc(me[wt] & ((1u << (t & 31)) - 1u));
          } else {  // slots before this one in token-major order with expert e
            for (int p = lane; p < f0 + q; p += 32) c += ids[p] == e;
          }
          c = warp_sum(c);
        }
        if (lane == 0) place(q, c);
      }
    }
    // token-in-rank entries of this CTA's tokens
    for (int q = tid; q < n_mine * R; q += kLayoutThreads) {
      const int t = first + q / R, r = q - (q / R) * R;
      int in = 0;
      for (int j = 0; j < k; ++j)
        in |= static_cast<unsigned>(ids[t * k + j] - r * G) < static_cast<unsigned>(G);
      a.in_rank[static_cast<long>(t) * R + r] = static_cast<uint8_t>(in);
    }
  } else if (n_mine > 0) {
    // ---- the first row (warps 8..): wait for it, cast it to FP8 ----
    ok = mbar_wait_bounded(&full[0], 0u, a.first_polls);
    if (kFp8 && ok) {
      cast_row(reinterpret_cast<const uint4 *>(in_buf), out_q, out_s, H, tid - kLayoutThreads,
               kCastThreads);
      fence_proxy_async_smem();  // the stage's generic writes before the bulk reads
    }
  }
  bool timed_out = __syncthreads_or(!ok);

  // 4. per token: (after the first) wait for its row and cast it, then k
  //    threads store it, one receive row each
  int i = 0;
  for (; i < n_mine && !timed_out; ++i) {
    const int s = i % kStages;
    if (i > 0) {
      ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kStages) & 1));
      if (__syncthreads_or(!ok)) {
        timed_out = true;
        break;
      }
      if (kFp8) {
        cast_row(reinterpret_cast<const uint4 *>(in_buf + s * in_bytes), out_q, out_s, H, tid,
                 kThreads);
        fence_proxy_async_smem();
        __syncthreads();
      }
    }
    if (tid < k) {
      // bf16: the stores read the bulk-loaded stage itself; their issuer
      // observes its completion (already passed, so this returns at once)
      if (!kFp8) mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kStages) & 1));
      const int row = rows[i * k + tid];
      if (row >= 0) {
        if (kFp8) {
          const int nb = H >> 7;
          bulk_store(a.recv + static_cast<long>(row) * H, out_q, H);
          bulk_store(a.recv_scale + static_cast<long>(row) * nb, out_s, 4 * nb);
        } else {
          bulk_store(a.recv + static_cast<long>(row) * in_bytes, in_buf + s * in_bytes, in_bytes);
        }
      }
      bulk_commit();
    }
    if (i + 1 < n_mine) {
      // the output stage (FP8) and input stage s (both) are read by the
      // stores: wait for that before they are overwritten
      if (tid < k) bulk_wait_read<0>();
      __syncthreads();
      if (tid == 0 && i + kStages < n_mine) issue(i + kStages);
    }
  }
  if (tid < k) bulk_wait_read<0>();  // stages read before the CTA exits
  if (tid == 0 && timed_out) {
    if (a.d_err != nullptr) atomicExch(reinterpret_cast<int *>(a.d_err), EP_ERR_TIMEOUT);
    // let the row loads still in flight land before the CTA's memory goes away
    for (int q = i; q < min(n_mine, i + kStages); ++q)
      mbar_wait_bounded(&full[q % kStages], static_cast<unsigned>((q / kStages) & 1));
  }
}

// ------------------------------------------------ one token per CTA

constexpr int kTokThreads = 1024;
constexpr int kTokWarps = kTokThreads / kWarp;
constexpr int kTokIdBatch = 4;  // ids per thread loaded before the cast

__host__ __device__ inline SmemMap token_smem_map(int T, int k, int E, int H, bool fp8) {
  SmemMap m;
  int o = 0;
  m.in = o;     o += 2 * H;
  m.out_q = o;  o += fp8 ? H : 0;
  m.out_s = o;  o += fp8 ? H / 32 : 0;
  m.mask = o;   // unused
  m.cnt = o;    o += align16(static_cast<long>(E) * 4);
  m.off = o;    o += align16(static_cast<long>(E + 1) * 4);
  m.cnt_r = o;  // unused: per-rank counts come from ballots
  m.ids = o;    o += align16(static_cast<long>(T) * k * 2);
  m.rows = o;
  m.total = o;
  return m;
}

__device__ __forceinline__ int valid_id(long long v, int E) {
  return v >= 0 && v < E ? static_cast<int>(v) : -1;
}

// out[0..n) = exclusive scan of in[0..n), out[n] = total, by all
// kTokThreads threads of the CTA.
__device__ void token_cta_exclusive_scan(const int *in, int *out, int n, int *warp_tot) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + kTokThreads - 1) / kTokThreads;
  const int b = min(n, tid * per), e = min(n, b + per);
  int local = 0;
  for (int q = b; q < e; ++q) local += in[q];
  const int incl = warp_incl_scan(local);
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < kTokWarps ? warp_tot[lane] : 0;
    const int iv = warp_incl_scan(v);
    if (lane < kTokWarps) warp_tot[lane] = iv - v;
    if (lane == kTokWarps - 1) out[n] = iv;
  }
  __syncthreads();
  int run = warp_tot[warp] + incl - local;
  for (int q = b; q < e; ++q) {
    out[q] = run;
    run += in[q];
  }
}

// Lets the next kernel on the stream be scheduled before this CTA exits
// (programmatic dependent launch).  Used only where a CTA's remaining work
// is its final stores: triggering earlier parks the next kernel's CTAs on
// SMs that are still busy.
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename IdT, bool kFp8>
__global__ void __launch_bounds__(kTokThreads) layout_dispatch_token_kernel(const FusedArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  const SmemMap sm = token_smem_map(a.T, a.k, a.E, a.H, kFp8);
  unsigned char *in_buf = smem + sm.in;
  uint2 *out_q = reinterpret_cast<uint2 *>(smem + sm.out_q);
  float *out_s = reinterpret_cast<float *>(smem + sm.out_s);
  int *cnt = reinterpret_cast<int *>(smem + sm.cnt);
  int *off = reinterpret_cast<int *>(smem + sm.off);
  int16_t *ids = reinterpret_cast<int16_t *>(smem + sm.ids);
  __shared__ __align__(8) uint64_t full;
  __shared__ int part[kTokWarps][EP_MAX_K];   // per-warp counts of smaller keys
  __shared__ int rpart[kTokWarps][EP_MAX_R];  // counts CTA: per-warp tokens per rank
  __shared__ int warp_tot[kTokWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int T = a.T, k = a.k, E = a.E, R = a.R, G = a.G, H = a.H;
  const int N = T * k;
  const int t = blockIdx.x;          // this CTA's token (t == T: the counts CTA)
  const bool counts_cta = t == T;
  const IdT *idx = static_cast<const IdT *>(a.idx);

  if (tid == 0 && !counts_cta) {
    mbar_init(&full, 1);
    mbar_init_fence();
  }
  if (counts_cta)
    for (int q = tid; q < E; q += kTokThreads) cnt[q] = 0;
  __syncthreads();  // barrier initialised and counters zeroed before use
  pdl_wait();       // ids and the row come from the previous kernel on the stream
  if (tid == 0 && !counts_cta) {
    mbar_arrive_expect_tx(&full, 2 * H);
    bulk_load(in_buf, a.x + static_cast<long>(t) * (H >> 3), 2 * H, &full);
  }

  // 1. ids into shared memory (validated: -1 for dropped and bad slots);
  //    a dispatch CTA casts its row to FP8 while the first batch is in flight
  long long v[kTokIdBatch];
#pragma unroll
  for (int u = 0; u < kTokIdBatch; ++u) {
    const int q = u * kTokThreads + tid;
    v[u] = q < N ? static_cast<long long>(idx[q]) : -1;
  }
  bool ok = true;
  if (!counts_cta) {
    ok = mbar_wait_bounded(&full, 0u, a.first_polls);
    if (kFp8 && ok) {
      cast_row(reinterpret_cast<const uint4 *>(in_buf), out_q, out_s, H, tid, kTokThreads);
      fence_proxy_async_smem();  // the stage's generic writes before the bulk reads
    }
  }
  auto take = [&](int q, long long raw) {
    const int e = valid_id(raw, E);
    ids[q] = static_cast<int16_t>(e);
    if (counts_cta) {
      if (e >= 0)
        atomicAdd(&cnt[e], 1);
      else if (raw != -1 && a.d_err != nullptr)
        atomicExch(reinterpret_cast<int *>(a.d_err), EP_ERR_INDEX);
    }
  };
#pragma unroll
  for (int u = 0; u < kTokIdBatch; ++u) {
    const int q = u * kTokThreads + tid;
    if (q < N) take(q, v[u]);
  }
  for (int q = kTokIdBatch * kTokThreads + tid; q < N; q += kTokThreads)
    take(q, static_cast<long long>(idx[q]));
  if (__syncthreads_or(!ok)) {
    if (tid == 0) {
      if (a.d_err != nullptr) atomicExch(reinterpret_cast<int *>(a.d_err), EP_ERR_TIMEOUT);
      mbar_wait_bounded(&full, 0u);  // let the row load land before the CTA exits
    }
    return;
  }

  if (counts_cta) {
    // 2c. the counts and offsets of the whole batch; tokens per rank as one
    //     ballot per rank and warp over the tokens' rank masks (R <= 64)
    if (lane == 0)
      for (int r = 0; r < R; ++r) rpart[warp][r] = 0;
    for (int t0 = 0; t0 < T; t0 += kTokThreads) {  // same trip count in every lane
      const int tt = t0 + tid;
      unsigned long long rm = 0ull;
      if (tt < T)
        for (int j = 0; j < k; ++j) {
          const int e = ids[tt * k + j];
          if (e >= 0) rm |= 1ull << ((static_cast<unsigned long long>(e) * a.g_magic) >> 32);
        }
      for (int r = 0; r < R; ++r) {
        const unsigned bal = __ballot_sync(0xffffffffu, ((rm >> r) & 1ull) != 0ull);
        if (lane == 0) rpart[warp][r] += __popc(bal);
      }
    }
    token_cta_exclusive_scan(cnt, off, E, warp_tot);
    __syncthreads();
    const int n_eff = off[E];
    for (int q = tid; q < E; q += kTokThreads) {
      a.cnt_e[q] = cnt[q];
      a.off_e[q] = off[q];
    }
    if (tid == 0) a.off_e[E] = n_eff;
    if (warp == kTokWarps - 1) {
      int carry = 0;
      for (int b = 0; b < R; b += 32) {
        const int r = b + lane;
        int c = 0;
        if (r < R)
          for (int v = 0; v < kTokWarps; ++v) c += rpart[v][r];
        const int incl = warp_incl_scan(c);
        if (r < R) {
          a.cnt_r[r] = c;
          a.off_r[r] = carry + incl - c;
        }
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) a.off_r[R] = carry;
    }
    for (int r = n_eff + tid; r < N; r += kTokThreads) a.recv_src[r] = -1;  // rows nobody fills
    return;
  }

  // 2d. receive rows of this token's k slots: count the smaller keys
  const int f0 = t * k;
  for (int j0 = 0; j0 < k; j0 += 8) {
    int ej[8], c[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      ej[jj] = j0 + jj < k ? ids[f0 + j0 + jj] : -1;
      c[jj] = 0;
    }
    for (int q = tid; q < N; q += kTokThreads) {
      const int e = ids[q];
      if (e < 0) continue;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        c[jj] += e < ej[jj] || (e == ej[jj] && q < f0 + j0 + jj);
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int sum = __reduce_add_sync(0xffffffffu, c[jj]);
      if (lane == 0 && j0 + jj < k) part[warp][j0 + jj] = sum;
    }
  }
  __syncthreads();

  // 3. layout entries of the token; lane j < k of warp 0 stores receive row j
  if (warp == 1) {
    for (int r = lane; r < R; r += 32) {
      int in = 0;
      for (int j = 0; j < k; ++j)
        in |= static_cast<unsigned>(ids[f0 + j] - r * G) < static_cast<unsigned>(G);
      a.in_rank[static_cast<long>(t) * R + r] = static_cast<uint8_t>(in);
    }
  }
  // nothing is left but the stores: the next kernel on the stream may be
  // scheduled now (it still waits for this grid's completion before it
  // reads anything), which hides its launch behind this CTA's stores
  // (decode call 8.22 -> 8.01 us in graphs of 20)
  pdl_trigger();
  if (warp == 0 && lane < k) {
    int before = 0;
    for (int v = 0; v < kTokWarps; ++v) before += part[v][lane];
    const int row = ids[f0 + lane] >= 0 ? before : -1;
    a.slot_pos[f0 + lane] = row;
    if (row >= 0) {
      a.recv_src[row] = t;
      if (kFp8) {
        const int nb = H >> 7;
        bulk_store(a.recv + static_cast<long>(row) * H, out_q, H);
        bulk_store(a.recv_scale + static_cast<long>(row) * nb, out_s, 4 * nb);
      } else {
        bulk_store(a.recv + static_cast<long>(row) * 2 * H, in_buf, 2 * H);
      }
      bulk_commit();
      bulk_wait_read<0>();  // the stage read before the CTA exits
    }
  }
}

template <typename IdT, bool kFp8>
cudaError_t launch_token_kernel(const FusedArgs &a, cudaStream_t s) {
  auto kern = layout_dispatch_token_kernel<IdT, kFp8>;
  const int smem = token_smem_map(a.T, a.k, a.E, a.H, kFp8).total;
  const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, dim3(a.T + 1), dim3(kTokThreads), smem, s, 1, a);
}

// CTAs of the token kernel that fit on `num_sms` SMs at once (0 = all).
template <typename IdT, bool kFp8>
long token_kernel_capacity(const FusedArgs &a, int num_sms) {
  const int smem = token_smem_map(a.T, a.k, a.E, a.H, kFp8).total;
  return persistent_grid(reinterpret_cast<const void *>(layout_dispatch_token_kernel<IdT, kFp8>),
                         kTokThreads, smem, 1L << 40, num_sms);
}

template <typename IdT, bool kFp8>
cudaError_t launch_fused(const FusedArgs &base, int num_sms, cudaStream_t s) {
  if (base.T + 1 <= token_kernel_capacity<IdT, kFp8>(base, num_sms))
    return launch_token_kernel<IdT, kFp8>(base, s);
  auto kern = layout_dispatch_kernel<IdT, kFp8>;
  // shared memory sized for ceil(T / SMs) tokens per CTA, which bounds the
  // tokens of a CTA below (at least one CTA per SM fits)
  const int sms = num_sms > 0 ? num_sms : device_sm_count();
  const int per_cta_max = (base.T + sms - 1) / sms;
  const int smem =
      smem_map(base.T, base.k, base.E, base.R, base.H, kFp8, per_cta_max).total;
  cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (err != cudaSuccess) return err;
  // a CTA per token, capped at the CTAs that fit at once; no CTA left empty
  const long cap = persistent_grid(reinterpret_cast<const void *>(kern), kThreads, smem,
                                   static_cast<long>(base.T) * (kThreads / kWarp), num_sms);
  FusedArgs a = base;
  a.per_cta = static_cast<int>((base.T + cap - 1) / cap);
  const int grid = (base.T + a.per_cta - 1) / a.per_cta;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, s, 1, a);
}

}  // namespace

bool layout_dispatch_fusable(int T, int k, int E, int R, int H, bool fp8,
                             const float *recv_scale) {
  (void)R;
  if (T < 1 || static_cast<long>(T) * k > kMaxSlots || H > kMaxH) return false;
  if (static_cast<long>(E) * ((T + 31) / 32) * 4 > kMaxMaskBytes) return false;
  if (fp8 && (H % 512 != 0 || reinterpret_cast<uintptr_t>(recv_scale) % 16 != 0)) return false;
  return true;
}

cudaError_t launch_layout_dispatch(const LayoutArgs &la, const void *x, int H, bool fp8,
                                   void *recv, float *recv_scale, int num_sms, cudaStream_t s,
                                   int *launches) {
  FusedArgs a{};
  a.idx = la.idx;
  a.T = la.T;
  a.k = la.k;
  a.E = la.E;
  a.R = la.R;
  a.G = la.E / la.R;
  a.g_magic = ((1ull << 32) + a.G - 1) / a.G;
  a.H = H;
  a.W = (la.T + 31) / 32;
  a.x = static_cast<const uint4 *>(x);
  a.cnt_e = la.cnt_e;
  a.cnt_r = la.cnt_r;
  a.off_e = la.off_e;
  a.off_r = la.off_r;
  a.slot_pos = la.slot_pos;
  a.recv_src = la.recv_src;
  a.in_rank = la.in_rank;
  a.recv = static_cast<unsigned char *>(recv);
  a.recv_scale = recv_scale;
  a.d_err = la.d_err;
  a.first_polls = first_wait_polls();
  ++*launches;
  if (la.id_kind == kIdsInt64)
    return fp8 ? launch_fused<long long, true>(a, num_sms, s)
               : launch_fused<long long, false>(a, num_sms, s);
  return fp8 ? launch_fused<int32_t, true>(a, num_sms, s)
             : launch_fused<int32_t, false>(a, num_sms, s);
}

}  // namespace ep
