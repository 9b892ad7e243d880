// layout.cu -- the dispatch layout on the GPU: per-expert and per-rank
// counts, the token-in-rank mask, exclusive prefix offsets and the stable
// receive row of every (token, slot).
//
// Three paths, all deterministic (no ordering ever depends on atomics):
//  * cluster (T*k below kGridMinSlots): one launch of a thread-block
//    cluster of up to 16 CTAs (a single plain CTA for small batches such as
//    a 128-token decode step).  Each CTA ranks its contiguous token range,
//    the CTAs exchange their per-expert counts through distributed shared
//    memory between two hardware cluster barriers, and every CTA then
//    places its own slots.  No global workspace.
//  * grid (kGridMinSlots <= T*k <= kClusterMaxSlots): the same per-CTA work
//    on one CTA per SM, launched cooperatively; the counts meet in the
//    caller's workspace between two grid barriers, the only waits of one
//    CTA on others in this library, each bounded.
//  * tiled (larger batches): a counting kernel writes one histogram row per
//    tile of tokens to the caller's workspace, and the last tile to finish
//    (ticket taken with atomicInc, which wraps it back to 0) turns the rows
//    into absolute per-tile bases and the global offsets; a placing kernel
//    then ranks and places every slot.
//
// Inside a CTA each warp owns a contiguous run of slots.  The lanes of a
// 32-slot chunk that hold the same expert find each other with one ballot
// per bit of the expert id (a slot's rank among them = popc of the lower
// such lanes); each warp keeps running per-expert counts in its own row of
// a shared histogram (row stride padded to avoid bank conflicts), and one
// thread per expert scans the rows across warps.  Slot order is therefore
// token-major order exactly.
#include <cooperative_groups.h>

#include <map>
#include <mutex>

#include "ep_internal.cuh"

namespace ep {
namespace {

namespace cg = cooperative_groups;

// CTA sizes of the cluster kernel: 512 threads while a CTA's slots fit the
// warps' registers (at most 4096 slots: 8 chunks of 32 per warp), which
// leaves room for 128 registers a thread; 1024 above that (64 registers).
// Measured at the prefill shape (2048 slots a CTA, 16 CTAs): 512 threads
// 9.2-9.5 us per launch after an L2 flush, 256 threads 10.5, 1024 threads
// 11.8-12.0; 3072 or 4096 slots a CTA (11 or 8 CTAs) 9.9-11.2 us.
constexpr int kClusterThreads = 1024;
constexpr int kClusterThreadsSmall = 512;
constexpr long kClusterSmallCtaSlots = 4096;
constexpr int kMaxClusterCtas = 16;
constexpr long kClusterMaxSlots = 1L << 19;
constexpr long kSlotsPerClusterCta = 2048;  // below this, fewer CTAs
constexpr long kSmallSlots = 2048;          // one CTA of kSmallThreads
constexpr int kSmallThreads = 256;

constexpr int kTileThreads = 512;
constexpr int kTileWarps = kTileThreads / kWarp;
constexpr int kTileTokensMin = 128;
constexpr int kMaxTiles = 296;  // 2 per SM on a 148-SM B200
constexpr int kTicketBytes = 16;

struct Params {
  const void *idx;
  int T, k, E, R;
  int id_bits;                 // bits of an expert id: 2^id_bits >= E
  unsigned long long g_magic;  // ceil(2^32 / G): e / G == (e * g_magic) >> 32 for e < 1024
  int32_t *cnt_e, *cnt_r, *off_e, *off_r, *slot_pos, *recv_src;
  uint8_t *in_rank;
  int32_t *d_err;
  unsigned *ticket;  // tiled path
  int32_t *cols;     // tiled path: [ntiles][E + R]
  int tile_T, ntiles;
  int stage;         // cluster / grid path: the CTA's checked ids live in shared memory
  unsigned *gbar;    // grid path: arrivals at barrier 1, at barrier 2, departures
  int first_polls;   // grid path: poll limit of the first barrier's wait
  int32_t *gcols;    // grid path: [E + R][CTAs] per-CTA counts, then their prefixes
  int32_t *gtot;     // grid path: [E + R] totals
};

// Expert id from a raw id value: -1 for a dropped or bad slot (a bad one
// is reported through d_err when given).
__device__ __forceinline__ int check_id(long long e, int E, int32_t *d_err) {
  if (e >= 0 && e < E) return static_cast<int>(e);
  if (e != -1 && d_err != nullptr) atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_INDEX);
  return -1;
}

__device__ __forceinline__ int rank_of(int e, const Params &p) {
  return static_cast<int>((static_cast<unsigned long long>(e) * p.g_magic) >> 32);
}

// Raw id of flat slot i.  int64 / int32 ids are read as they are; a uint8
// token-in-rank mask [T, k] is read as "slot (t, r) belongs to expert r"
// (r = i % k) when set, else dropped -- the rank-row layout is the expert
// layout of that mask.
template <typename IdT>
__device__ __forceinline__ long long raw_id(const IdT *idx, long i, int /*k*/) {
  return static_cast<long long>(idx[i]);
}
template <>
__device__ __forceinline__ long long raw_id<uint8_t>(const uint8_t *idx, long i, int k) {
  return idx[i] ? static_cast<long long>(static_cast<unsigned>(i) % static_cast<unsigned>(k)) : -1;
}

// Token of flat slot i: slots number fewer than 2^31, so the 32-bit
// unsigned division is exact and far cheaper than a 64-bit one.
__device__ __forceinline__ int32_t token_of_slot(long i, int k) {
  return static_cast<int32_t>(static_cast<unsigned>(i) / static_cast<unsigned>(k));
}

// Ids are read kIdBatch at a time per lane, all loads issued before any is
// used, so a warp pays one memory round trip per kIdBatch * 32 slots.
constexpr int kIdBatch = 8;

template <typename IdT>
__device__ __forceinline__ void load_id_batch(const IdT *idx, long c0, long end, int k,
                                              long long (&v)[kIdBatch]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < kIdBatch; ++b) {
    const long i = c0 + 32 * b + lane;
    v[b] = i < end ? raw_id(idx, i, k) : -1;
  }
}

// Contiguous, 32-aligned slice [b, *end) of [0, n) for warp w of nw.
__device__ __forceinline__ long warp_slice(long n, int w, int nw, long *end) {
  const long s = ((n + nw - 1) / nw + 31) / 32 * 32;
  const long b = min(n, s * w);
  *end = min(n, b + s);
  return b;
}

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Exclusive scan of a[0..n) in shared memory by one warp, 32 consecutive
// elements per round (conflict-free); returns the total to every lane.
__device__ int warp_exclusive_scan_smem(int *a, int n) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int x = i < n ? a[i] : 0;
    const int incl = warp_inclusive_scan(x);
    if (i < n) a[i] = carry + incl - x;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  return carry;
}

// Lanes of the warp whose key equals this lane's, among the lanes in
// `valid`: the intersection over the key's bits of the lanes that agree on
// each bit (one ballot per bit).
__device__ __forceinline__ unsigned match_key(int key, int bits, unsigned valid) {
  unsigned peers = valid;
  for (int b = 0; b < bits; ++b) {
    const unsigned ones = __ballot_sync(0xffffffffu, (key >> b) & 1);
    peers &= ((key >> b) & 1) ? ones : ~ones;
  }
  return peers;
}

// Per-warp histograms: row w holds warp w's counts, columns [0, E) experts
// and [E, E + R) ranks; the row stride E + R + 1 keeps the threads of one
// column scan on distinct banks.
__device__ __forceinline__ int hist_ld(const Params &p) { return p.E + p.R + 1; }

// For each column c of the nw rows, one thread: hist[w][c] becomes the
// count of the earlier warps (experts only) and total[c] the CTA's count.
__device__ void scan_hist_columns(int *hist, int ld, int E, int C, int nw, int *total) {
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    int run = 0;
    for (int v = 0; v < nw; ++v) {
      const int x = hist[v * ld + c];
      if (c < E) hist[v * ld + c] = run;
      run += x;
    }
    total[c] = run;
  }
}

// hist[w][e] += base[e] for every warp w (base: the expert's first row for
// this CTA), one thread per expert.
__device__ void add_column_bases(int *hist, int ld, int E, int nw, const int *base) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int b = base[e];
    for (int v = 0; v < nw; ++v) hist[v * ld + e] += b;
  }
}

// A warp's stable ranking of its slot segment [beg, end).
//
// Pass 1 (rank_segment) walks the segment 32 slots at a time: a slot's rank
// among the warp's slots of its expert is the warp's running count of that
// expert (hist_w[e], zeroed by the caller) plus the number of lower lanes
// holding the same expert.  The first kRegChunks chunks keep expert and
// rank in registers (packed as rank << 10 | e, -1 for no kept slot; E <=
// 1024); later chunks park the rank in the slot_pos output.  At the end
// hist_w[e] is the warp's count of e.
//
// Pass 2 (place_segment) turns ranks into rows, base_w[e] being the
// warp's first row of expert e, and writes slot_pos and recv_src.
constexpr int kRegChunks = kIdBatch;

struct SegRanks {
  int packed[kRegChunks];
};

__device__ __forceinline__ int rank_one(int e, int bits, int *hist_w) {
  const unsigned lt = lanemask_lt();
  const unsigned valid = __ballot_sync(0xffffffffu, e >= 0);
  const unsigned peers = match_key(e, bits, valid);
  const int r = e >= 0 ? hist_w[e] + __popc(peers & lt) : -1;
  __syncwarp();
  if (e >= 0 && (peers & lt) == 0) hist_w[e] += __popc(peers);
  __syncwarp();
  return r;
}

// Slots past the register chunks (CTA shares above 32 * kRegChunks slots
// a warp), out of line: code a launch does not run stays out of the way of
// the code it does, which the SMs fetch cold after the caches are flushed
// (prefill layout 13.2 -> 9.5 us a launch after a flush, 8.8 -> 8.6 warm).
template <typename IdT>
__device__ __noinline__ void rank_rest(const IdT *idx, long from, long end, int k, int E, int bits,
                                       int32_t *d_err, int *hist_w, int32_t *slot_pos,
                                       short *ids_smem, long cta_beg) {
  const int lane = threadIdx.x & 31;
  for (long c0 = from; c0 < end; c0 += 32 * kIdBatch) {
    long long v[kIdBatch];
    load_id_batch(idx, c0, end, k, v);
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      if (c0 + 32 * b >= end) break;  // uniform across the warp
      const long i = c0 + 32 * b + lane;
      const int e = check_id(v[b], E, d_err);
      const int r = rank_one(e, bits, hist_w);
      if (i < end) {
        slot_pos[i] = r;
        if (ids_smem != nullptr) ids_smem[i - cta_beg] = static_cast<short>(e);
      }
    }
  }
}

// ids_smem (optional): the checked ids of the CTA's slots, indexed from
// cta_beg, for the token-mask pass to read from shared memory.
template <typename IdT>
__device__ void rank_segment(const IdT *idx, long beg, long end, const Params &p,
                             int32_t *d_err, int *hist_w, int32_t *slot_pos, SegRanks &sr,
                             short *ids_smem = nullptr, long cta_beg = 0) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, bits = p.id_bits;
  {
    long long v[kIdBatch];
    load_id_batch(idx, beg, end, p.k, v);
#pragma unroll
    for (int b = 0; b < kRegChunks; ++b) {
      sr.packed[b] = -1;
      if (beg + 32 * b < end) {  // uniform across the warp
        const int e = check_id(v[b], E, d_err);
        const int r = rank_one(e, bits, hist_w);
        sr.packed[b] = e >= 0 ? (r << 10) | e : -1;
        const long i = beg + 32 * b + lane;
        if (ids_smem != nullptr && i < end) ids_smem[i - cta_beg] = static_cast<short>(e);
      }
    }
  }
  if (beg + 32 * kRegChunks < end)
    rank_rest(idx, beg + 32 * kRegChunks, end, p.k, E, bits, d_err, hist_w, slot_pos, ids_smem,
              cta_beg);
}

// The first row of expert e for this warp: base_w[e] (+ add1[e] + add2[e]
// when given: the CTA's offset in the expert and the expert's offset).
__device__ __forceinline__ int warp_base(int e, const int *base_w, const int *add1,
                                         const int *add2) {
  int b = base_w[e];
  if (add1 != nullptr) b += add1[e] + add2[e];
  return b;
}

// place_segment's counterpart of rank_rest, out of line for the same reason.
template <typename IdT>
__device__ __noinline__ void place_rest(const IdT *idx, long from, long end, int k, int E,
                                        const int *base_w, int32_t *slot_pos, int32_t *recv_src,
                                        const int *add1, const int *add2) {
  const int lane = threadIdx.x & 31;
  for (long c0 = from; c0 < end; c0 += 32 * kIdBatch) {
    long long v[kIdBatch];
    load_id_batch(idx, c0, end, k, v);
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const long i = c0 + 32 * b + lane;
      if (i < end) {
        const int e = check_id(v[b], E, nullptr);
        const int pos = e >= 0 ? warp_base(e, base_w, add1, add2) + slot_pos[i] : -1;
        slot_pos[i] = pos;
        if (pos >= 0) recv_src[pos] = token_of_slot(i, k);
      }
    }
  }
}

template <typename IdT>
__device__ void place_segment(const IdT *idx, long beg, long end, int k, int E,
                              const int *base_w, const SegRanks &sr, int32_t *slot_pos,
                              int32_t *recv_src, const int *add1 = nullptr,
                              const int *add2 = nullptr) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < kRegChunks; ++b) {
    const long i = beg + 32 * b + lane;
    if (i < end) {
      const int q = sr.packed[b];
      const int pos = q >= 0 ? warp_base(q & 1023, base_w, add1, add2) + (q >> 10) : -1;
      slot_pos[i] = pos;
      if (pos >= 0) recv_src[pos] = token_of_slot(i, k);
    }
  }
  if (beg + 32 * kRegChunks < end)
    place_rest(idx, beg + 32 * kRegChunks, end, k, E, base_w, slot_pos, recv_src, add1, add2);
}

// Bit r set when token t has a kept slot in rank r, from the ids in
// global memory (the CTAs whose ids are not staged in shared memory), out
// of line as rank_rest is.
template <typename IdT>
__device__ __noinline__ unsigned long long token_rank_bits(const IdT *idx, int t, int k, int E,
                                                           unsigned long long g_magic) {
  const long base = static_cast<long>(t) * k;
  unsigned long long m = 0;
  for (int j0 = 0; j0 < k; j0 += kIdBatch) {
    long long v[kIdBatch];
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) v[b] = j0 + b < k ? raw_id(idx, base + j0 + b, k) : -1;
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int e = check_id(v[b], E, nullptr);
      if (e >= 0) m |= 1ull << ((static_cast<unsigned long long>(e) * g_magic) >> 32);
    }
  }
  return m;
}

// Token-in-rank mask rows for tokens [t_beg, t_end).  Per-rank token counts
// go into this warp's histogram row, columns E..E+R-1 (one ballot per rank,
// written by lane 0: the row is the warp's own).  Every thread of the
// block runs the same number of rounds.
template <typename IdT>
__device__ void rank_mask(const Params &p, int t_beg, int t_end, int *hist_w,
                          const short *ids_smem = nullptr) {
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int lane = threadIdx.x & 31;
  for (int t0 = t_beg; t0 < t_end; t0 += blockDim.x) {
    const int t = t0 + threadIdx.x;
    unsigned long long m = 0;
    if (t < t_end && ids_smem != nullptr) {
      const short *ids = ids_smem + static_cast<long>(t - t_beg) * p.k;
      for (int j = 0; j < p.k; ++j) {
        const int e = ids[j];
        if (e >= 0) m |= 1ull << rank_of(e, p);
      }
    } else if (t < t_end) {
      m = token_rank_bits(idx, t, p.k, p.E, p.g_magic);
    }
    if (t < t_end && p.in_rank != nullptr) {
      uint8_t *row = p.in_rank + static_cast<long>(t) * p.R;
      if ((p.R & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 3) == 0) {
        // 4 mask bytes per 32-bit store
        for (int r = 0; r < p.R; r += 4) {
          const unsigned b = static_cast<unsigned>(m >> r);
          reinterpret_cast<uint32_t *>(row)[r >> 2] =
              (b & 1u) | ((b >> 1) & 1u) << 8 | ((b >> 2) & 1u) << 16 | ((b >> 3) & 1u) << 24;
        }
      } else {
        for (int r = 0; r < p.R; ++r) row[r] = static_cast<uint8_t>((m >> r) & 1u);
      }
    }
    for (int r = 0; r < p.R; ++r) {
      const unsigned bal = __ballot_sync(0xffffffffu, (m >> r) & 1u);
      if (lane == 0) hist_w[p.E + r] += __popc(bal);
    }
  }
}

// ------------------------------------------------------------- cluster path

// Split cluster barrier: every thread of every CTA arrives once at kernel
// start, and waits before its first access to another CTA's shared memory,
// which is then guaranteed to be running.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
}

// Slots per CTA up to which the CTA's checked ids are kept in shared
// memory (int16) for the token-mask pass, when that fits.
constexpr long kStageIdsMax = 16384;

// Shared memory of the cluster kernel: per-warp histograms, every CTA's
// counts, the lower CTAs' counts, the totals, and (staged) the CTA's
// checked ids (int16).
int cluster_smem_bytes(int E, int R, int warps, int ctas, long staged) {
  return (warps * (E + R + 1) + (ctas + 2) * (E + R)) * static_cast<int>(sizeof(int)) +
         static_cast<int>(((staged * 2 + 15) / 16) * 16);
}

// Warp-wide exclusive scan of a[0..n) in place (32 elements per round) that
// also writes the counts (cnt) and the exclusive offsets plus the total at
// off[n] when those are given; returns the total.
__device__ int scan_counts(int *a, int n, int32_t *cnt, int32_t *off) {
  const int lane = threadIdx.x & 31;
  int carry = 0;
  for (int base = 0; base < n; base += 32) {
    const int i = base + lane;
    const int x = i < n ? a[i] : 0;
    const int incl = warp_inclusive_scan(x);
    if (i < n) {
      a[i] = carry + incl - x;
      if (cnt != nullptr) cnt[i] = x;
      if (off != nullptr) off[i] = carry + incl - x;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (off != nullptr && lane == 0) off[n] = carry;
  return carry;
}

// Exclusive scans, in place and by every thread of the CTA, of a[0..n)
// and (when b is given) b[0..n), n <= 1024: each warp scans 32-entry
// chunks, then warps 0 and 1 scan the chunk sums (no serial chain through
// all n entries).  cnt / off, when given, receive a's entries and
// exclusive offsets (off[n] = the total).  Warp 2 meanwhile scans the nr
// rank totals r[] (cnt_r / off_r when given).  Returns a's total (and b's
// in *b_total).  wsum: 66 ints of shared scratch.  Holds three CTA
// barriers.
__device__ int block_scan_counts(int *a, int *b, int n, int32_t *cnt, int32_t *off, int *r,
                                 int nr, int32_t *cnt_r, int32_t *off_r, int *wsum,
                                 int *b_total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int nch = (n + 31) / 32;
  for (int c = w; c < nch; c += nw) {
    const int i = c * 32 + lane;
    const int x = i < n ? a[i] : 0;
    const int ix = warp_inclusive_scan(x);
    if (i < n) {
      a[i] = ix - x;
      if (cnt != nullptr) cnt[i] = x;
    }
    if (lane == 31) wsum[c] = ix;
    if (b != nullptr) {
      const int y = i < n ? b[i] : 0;
      const int iy = warp_inclusive_scan(y);
      if (i < n) b[i] = iy - y;
      if (lane == 31) wsum[32 + c] = iy;
    }
  }
  __syncthreads();
  if (w == 0 || (w == 1 && b != nullptr)) {
    int *ws = wsum + 32 * w;
    const int v = lane < nch ? ws[lane] : 0;
    const int iv = warp_inclusive_scan(v);
    if (lane < nch) ws[lane] = iv - v;
    if (lane == 31) {
      wsum[64 + w] = iv;
      if (w == 0 && off != nullptr) off[n] = iv;
    }
  } else if (w == 2) {
    scan_counts(r, nr, cnt_r, off_r);
  }
  __syncthreads();
  for (int c = w; c < nch; c += nw) {
    const int i = c * 32 + lane;
    if (i < n) {
      a[i] += wsum[c];
      if (off != nullptr) off[i] = a[i];
      if (b != nullptr) b[i] += wsum[32 + c];
    }
  }
  const int total = wsum[64];
  if (b_total != nullptr) *b_total = b != nullptr ? wsum[65] : 0;
  __syncthreads();
  return total;
}

template <typename IdT, int kThreads>
__global__ void __launch_bounds__(kThreads, 1) layout_cluster_kernel(Params p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int n_ctas = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  if (n_ctas > 1) cluster_arrive_relaxed();
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R, ld = hist_ld(p);
  const int tid = threadIdx.x, nt = blockDim.x, w = tid >> 5, nw = nt >> 5;
  int *hist = smem;                // [warps][E + R + 1]
  int *all = hist + nw * ld;       // [ctas][C] every CTA's counts, pushed by each CTA
  int *before = all + n_ctas * C;  // [C] counts of the lower-ranked CTAs
  int *tot = before + C;           // [C] totals, then exclusive offsets
  short *ids_smem = reinterpret_cast<short *>(tot + C);  // staged ids
  __shared__ int wsum[66];
  const IdT *idx = static_cast<const IdT *>(p.idx);

  const int per_cta = (p.T + n_ctas - 1) / n_ctas;
  const int t_beg = min(p.T, rank * per_cta);
  const int t_end = min(p.T, t_beg + per_cta);
  const long s_beg = static_cast<long>(t_beg) * p.k;
  const long n = static_cast<long>(t_end - t_beg) * p.k;
  const bool stage = p.stage != 0;

  for (int i = tid; i < nw * ld; i += nt) smem[i] = 0;
  __syncthreads();
  pdl_wait();
  long seg_end;
  const long seg_beg = warp_slice(n, w, nw, &seg_end);
  SegRanks sr;
  rank_segment(idx, s_beg + seg_beg, s_beg + seg_end, p, p.d_err, hist + w * ld, p.slot_pos,
               sr, stage ? ids_smem : nullptr, s_beg);
  if (stage) __syncthreads();  // every warp's ids are in shared memory
  rank_mask<IdT>(p, t_beg, t_end, hist + w * ld, stage ? ids_smem : nullptr);
  __syncthreads();
  if (n_ctas > 1) cluster_wait();  // every CTA of the cluster is running
  // one thread per column: exclusive prefix over this CTA's warps; the
  // CTA's count goes to row `rank` of every CTA's `all` (or straight to
  // `tot` when the CTA is alone)
  for (int c = tid; c < C; c += nt) {
    int run = 0;
    for (int v = 0; v < nw; ++v) {
      const int x = hist[v * ld + c];
      if (c < E) hist[v * ld + c] = run;
      run += x;
    }
    if (n_ctas > 1) {
      for (int q = 0; q < n_ctas; ++q) cluster.map_shared_rank(all, q)[rank * C + c] = run;
    } else {
      before[c] = 0;
      tot[c] = run;
    }
  }
  if (n_ctas > 1) {
    cluster.sync();  // all pushes done and visible; nothing remote after this
    for (int c = tid; c < C; c += nt) {
      int b = 0, a = 0;
      for (int r = 0; r < n_ctas; ++r) {
        const int v = all[r * C + c];
        b += r < rank ? v : 0;
        a += v;
      }
      before[c] = b;
      tot[c] = a;
    }
  }
  __syncthreads();
  // exclusive scans of the expert totals (their offsets; CTA 0 writes
  // them with the counts) and of the rank totals
  const int n_kept = block_scan_counts(
      tot, nullptr, E, rank == 0 ? p.cnt_e : nullptr, rank == 0 ? p.off_e : nullptr, tot + E, R,
      rank == 0 ? p.cnt_r : nullptr, rank == 0 ? p.off_r : nullptr, wsum, nullptr);
  // row = this warp's count of earlier slots + the CTA's offset in the
  // expert (before) + the expert's offset (tot)
  place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * ld, sr, p.slot_pos,
                p.recv_src, before, tot);
  // rows nobody fills (past the kept ones)
  const long N = static_cast<long>(p.T) * p.k;
  for (long r = n_kept + static_cast<long>(rank) * nt + tid; r < N;
       r += static_cast<long>(n_ctas) * nt)
    p.recv_src[r] = -1;
}

// ------------------------------------------------------------- grid path
//
// Mid-size batches on every SM instead of one cluster's 16: one CTA of
// kGridThreads per SM, launched cooperatively so that all of them run at
// once, each ranking a contiguous token range as a cluster CTA does.  The
// per-CTA counts meet in the workspace: after a first grid barrier, CTA c
// scans columns c, c + G, ... of the [E + R][G] count matrix over the CTAs
// (exclusive, in place) and writes their totals; after a second barrier
// every CTA reads its own prefixes and the totals and places its slots.
// Both barriers are bounded waits (EP_ERR_TIMEOUT in d_err when one gives
// up); the last CTA to leave sets the barrier counters back to zero.
constexpr int kGridThreads = 512;
constexpr int kGridMaxCtas = 160;               // the workspace is sized for this many
constexpr size_t kGridHeaderBytes = 16;            // three counters, padded
constexpr size_t kGridMaxWsBytes = 256u << 10;     // larger E + R: the cluster kernel
constexpr int kMaxGridPolls = 1 << 20;             // x ~0.1 us of sleep each

// Arrive at the grid barrier counter `ctr` and wait, polling at most
// `max_polls` times, until all `n_ctas` CTAs have; false when the wait gave
// up.  Every thread of every CTA must call it.
__device__ bool grid_sync(unsigned *ctr, unsigned n_ctas, int max_polls, int *s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's writes before its arrival
    atomicAdd(ctr, 1u);
    int ok = 1;
    for (int polls = 0; *reinterpret_cast<volatile unsigned *>(ctr) < n_ctas; ++polls) {
      if (polls >= max_polls) {
        ok = 0;
        break;
      }
      __nanosleep(100);
    }
    __threadfence();  // the other CTAs' writes after their arrivals
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

int grid_smem_bytes(int E, int R, long staged) {
  return ((kGridThreads / kWarp) * (E + R + 1) + 2 * (E + R)) * static_cast<int>(sizeof(int)) +
         static_cast<int>(((staged * 2 + 15) / 16) * 16);
}

template <typename IdT>
__global__ void __launch_bounds__(kGridThreads, 1) layout_grid_kernel(Params p) {
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R, ld = hist_ld(p);
  const int tid = threadIdx.x, lane = tid & 31, nt = blockDim.x, w = tid >> 5, nw = nt >> 5;
  const int G = gridDim.x, cta = blockIdx.x;
  int *hist = smem;              // [warps][E + R + 1]
  int *before = hist + nw * ld;  // [C] counts of the lower CTAs
  int *tot = before + C;         // [C] totals, then exclusive offsets
  short *ids_smem = reinterpret_cast<short *>(tot + C);  // staged ids
  __shared__ int wsum[66];
  __shared__ int s_ok;
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const bool stage = p.stage != 0;

  const int t_beg = static_cast<int>(static_cast<long>(p.T) * cta / G);
  const int t_end = static_cast<int>(static_cast<long>(p.T) * (cta + 1) / G);
  const long s_beg = static_cast<long>(t_beg) * p.k;
  const long n = static_cast<long>(t_end - t_beg) * p.k;

  for (int i = tid; i < nw * ld; i += nt) hist[i] = 0;
  __syncthreads();
  pdl_wait();
  long seg_end;
  const long seg_beg = warp_slice(n, w, nw, &seg_end);
  SegRanks sr;
  rank_segment(idx, s_beg + seg_beg, s_beg + seg_end, p, p.d_err, hist + w * ld, p.slot_pos,
               sr, stage ? ids_smem : nullptr, s_beg);
  if (stage) __syncthreads();  // every warp's ids are in shared memory
  rank_mask<IdT>(p, t_beg, t_end, hist + w * ld, stage ? ids_smem : nullptr);
  __syncthreads();
  // one thread per column: exclusive prefix over this CTA's warps; the
  // CTA's count goes to its slot of the column in the workspace
  for (int col = tid; col < C; col += nt) {
    int run = 0;
    for (int v = 0; v < nw; ++v) {
      const int x = hist[v * ld + col];
      if (col < E) hist[v * ld + col] = run;
      run += x;
    }
    p.gcols[static_cast<long>(col) * G + cta] = run;
  }
  bool ok = grid_sync(&p.gbar[0], G, p.first_polls, &s_ok);
  if (ok) {
    // columns cta, cta + G, ...: one warp each, exclusive over the CTAs;
    // the whole column (G <= kGridMaxCtas values) is loaded before any of
    // it is scanned, so that it costs one round trip to L2
    constexpr int kPer = (kGridMaxCtas + 31) / 32;
    for (int col = cta + G * w; col < C; col += G * nw) {
      int32_t *colp = p.gcols + static_cast<long>(col) * G;
      int x[kPer];
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = 32 * j + lane;
        x[j] = i < G ? __ldcg(colp + i) : 0;
      }
      int carry = 0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int i = 32 * j + lane;
        const int incl = warp_inclusive_scan(x[j]);
        if (i < G) colp[i] = carry + incl - x[j];
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) p.gtot[col] = carry;
    }
  }
  ok = grid_sync(&p.gbar[1], G, kMaxGridPolls, &s_ok) && ok;
  if (ok) {
    for (int col = tid; col < C; col += nt) {
      before[col] = __ldcg(p.gcols + static_cast<long>(col) * G + cta);
      tot[col] = __ldcg(p.gtot + col);
    }
    __syncthreads();
    // exclusive scans of the expert totals (their offsets; CTA 0 writes
    // them with the counts) and of the rank totals
    const int n_kept = block_scan_counts(
        tot, nullptr, E, cta == 0 ? p.cnt_e : nullptr, cta == 0 ? p.off_e : nullptr, tot + E,
        R, cta == 0 ? p.cnt_r : nullptr, cta == 0 ? p.off_r : nullptr, wsum, nullptr);
    place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * ld, sr,
                  p.slot_pos, p.recv_src, before, tot);
    // rows nobody fills (past the kept ones)
    const long N = static_cast<long>(p.T) * p.k;
    for (long r = n_kept + static_cast<long>(cta) * nt + tid; r < N;
         r += static_cast<long>(G) * nt)
      p.recv_src[r] = -1;
  } else if (tid == 0 && p.d_err != nullptr) {
    atomicExch(reinterpret_cast<int *>(p.d_err), EP_ERR_TIMEOUT);
  }
  // every CTA is past both barriers once all have left: the last one out
  // sets the counters back to zero for the next call on this workspace
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.gbar[2], 1u) == static_cast<unsigned>(G - 1)) {
      p.gbar[0] = 0u;
      p.gbar[1] = 0u;
      p.gbar[2] = 0u;
      __threadfence();
    }
  }
}

// ------------------------------------------------------------- tiled path

template <typename IdT>
__global__ void __launch_bounds__(kTileThreads) layout_count_kernel(Params p) {
  pdl_wait();
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R, ld = hist_ld(p);
  const int tid = threadIdx.x, nt = blockDim.x, w = tid >> 5, nw = nt >> 5;
  int *hist = smem;                   // [warps][E + R + 1] per-warp counts
  int *col = hist + nw * ld;          // [C] this tile's counts, later totals
  int *part = col + C;                // [max(nt, C)] partial column sums
  int *flag = part + max(nt, C);      // [1]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tile = blockIdx.x;
  const int t_beg = tile * p.tile_T;
  const int t_end = min(p.T, t_beg + p.tile_T);

  for (int i = tid; i < nw * ld; i += nt) hist[i] = 0;
  __syncthreads();
  const long s_end = static_cast<long>(t_end) * p.k;
  for (long c0 = static_cast<long>(t_beg) * p.k; c0 < s_end;
       c0 += static_cast<long>(nt) * kIdBatch) {
    long long v[kIdBatch];
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const long i = c0 + static_cast<long>(b) * nt + tid;
      v[b] = i < s_end ? raw_id(idx, i, p.k) : -1;
    }
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int e = check_id(v[b], E, p.d_err);
      if (e >= 0) atomicAdd(&hist[w * ld + e], 1);
    }
  }
  rank_mask<IdT>(p, t_beg, t_end, hist + w * ld);
  __syncthreads();
  scan_hist_columns(hist, ld, E, C, nw, col);
  __syncthreads();
  for (int c = tid; c < C; c += nt) p.cols[static_cast<long>(tile) * C + c] = col[c];

  // the last tile to get here finishes the scan for everyone
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned ticket = atomicInc(p.ticket, p.ntiles - 1);
    flag[0] = (ticket == static_cast<unsigned>(p.ntiles - 1));
  }
  __syncthreads();
  if (!flag[0]) return;
  __threadfence();

  // column totals, each column split into P contiguous runs of tiles; loads
  // go out 8 at a time
  const int P = max(1, nt / C);
  const int chunk = (p.ntiles + P - 1) / P;
  for (int q = tid; q < C * P; q += nt) {
    const int c = q % C, pp = q / C;
    const int b = pp * chunk, e_ = min(p.ntiles, b + chunk);
    int s = 0;
    for (int tl = b; tl < e_; tl += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = tl + u < e_ ? __ldcg(&p.cols[static_cast<long>(tl + u) * C + c]) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) s += v[u];
    }
    part[pp * C + c] = s;
  }
  __syncthreads();
  for (int c = tid; c < C; c += nt) {
    int s = 0;
    for (int pp = 0; pp < P; ++pp) s += part[pp * C + c];
    col[c] = s;
    if (c < E) p.cnt_e[c] = s;
    else if (p.cnt_r != nullptr) p.cnt_r[c - E] = s;
  }
  __syncthreads();
  if (w == 0) {
    const int n_kept = warp_exclusive_scan_smem(col, E);
    if (tid == 0) p.off_e[E] = n_kept;
  } else if (w == 1) {
    const int n_tok = warp_exclusive_scan_smem(col + E, R);
    if ((tid & 31) == 0 && p.off_r != nullptr) p.off_r[R] = n_tok;
  }
  __syncthreads();
  for (int c = tid; c < C; c += nt) {
    if (c < E) p.off_e[c] = col[c];
    else if (p.off_r != nullptr) p.off_r[c - E] = col[c];
  }
  // absolute row base of every (tile, expert), in place
  for (int q = tid; q < C * P; q += nt) {
    const int c = q % C, pp = q / C;
    if (c >= E) continue;
    int base = col[c];
    for (int v = 0; v < pp; ++v) base += part[v * C + c];
    const int b = pp * chunk, e_ = min(p.ntiles, b + chunk);
    for (int tl = b; tl < e_; tl += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        v[u] = tl + u < e_ ? __ldcg(&p.cols[static_cast<long>(tl + u) * C + c]) : 0;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (tl + u < e_) {
          p.cols[static_cast<long>(tl + u) * C + c] = base;
          base += v[u];
        }
    }
  }
}

template <typename IdT>
__global__ void __launch_bounds__(kTileThreads) layout_place_kernel(Params p) {
  pdl_wait();
  // every count tile is done with the ticket: leave it at zero for the next
  // call on this workspace, whatever value it has (a completed count kernel
  // leaves zero anyway, through the wrap of atomicInc; two calls that
  // overlapped on one workspace might not)
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.ticket = 0u;
  extern __shared__ int smem[];
  const int E = p.E, C = p.E + p.R, ld = hist_ld(p);
  const int tid = threadIdx.x, w = tid >> 5;
  int *hist = smem;                    // [warps][E + R + 1]
  int *base = hist + kTileWarps * ld;  // [E] the tile's first row of each expert
  int *scratch = base + E;             // [C] tile totals (unused)
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tile = blockIdx.x;
  const int t_beg = tile * p.tile_T;
  const int t_end = min(p.T, t_beg + p.tile_T);
  const long s_beg = static_cast<long>(t_beg) * p.k;
  const long n = static_cast<long>(t_end - t_beg) * p.k;

  for (int i = tid; i < kTileWarps * ld; i += blockDim.x) hist[i] = 0;
  for (int e = tid; e < E; e += blockDim.x)
    base[e] = __ldcg(&p.cols[static_cast<long>(tile) * C + e]);
  __syncthreads();
  long seg_end;
  const long seg_beg = warp_slice(n, w, kTileWarps, &seg_end);
  SegRanks sr;
  rank_segment(idx, s_beg + seg_beg, s_beg + seg_end, p, nullptr, hist + w * ld, p.slot_pos,
               sr);
  __syncthreads();
  scan_hist_columns(hist, ld, E, E, kTileWarps, scratch);
  __syncthreads();
  add_column_bases(hist, ld, E, kTileWarps, base);
  __syncthreads();
  place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * ld, sr, p.slot_pos,
                p.recv_src);

  // rows nobody fills
  const long N = static_cast<long>(p.T) * p.k;
  const long n_kept = __ldcg(&p.off_e[E]);
  for (long r = n_kept + static_cast<long>(blockIdx.x) * blockDim.x + tid; r < N;
       r += static_cast<long>(gridDim.x) * blockDim.x)
    p.recv_src[r] = -1;
}

// ---------------------------------------------------------------- launch

int tile_tokens(int T) {
  const int t = (T + kMaxTiles - 1) / kMaxTiles;
  return t > kTileTokensMin ? t : kTileTokensMin;
}

bool cluster_path(int T, int k) { return static_cast<long>(T) * k <= kClusterMaxSlots; }

// Batches from this many slots up to kClusterMaxSlots take the grid
// kernel when its workspace is small enough.  Its fixed cost (about 12 us
// a launch in CUDA graphs, whatever the size) is above the cluster
// kernel's below that: 11.7 against 8.8 us at 32768 slots, even at 65536
// (12.0 / 11.3 warm, 16.2 / 16.9 after a flush), 12.0 against 18.0 at
// 131072 and 13.9 against 31.9 at 262144.
constexpr long kGridMinSlots = 65536;

int grid_ctas() { return min(device_sm_count(), kGridMaxCtas); }

// Workspace of the grid kernel, sized for kGridMaxCtas CTAs so that it
// does not depend on the device.
size_t grid_ws_bytes(int E, int R) {
  const size_t C = static_cast<size_t>(E) + R;
  return kGridHeaderBytes + (C * kGridMaxCtas + C) * sizeof(int32_t);
}

bool grid_path(int T, int k, int E, int R) {
  const long N = static_cast<long>(T) * k;
  return N >= kGridMinSlots && N <= kClusterMaxSlots && grid_ws_bytes(E, R) <= kGridMaxWsBytes;
}

// Largest cluster (<= 16 CTAs) the device can schedule for this kernel with
// `smem` bytes per CTA; cached per (device, id type, smem size).
// Largest cluster (16, else the portable 8) the GPU can run with CTAs of
// kThreads threads and `smem` bytes of dynamic shared memory.
template <typename IdT, int kThreads>
int max_cluster_ctas(int smem) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, smem});
  if (it != cache.end()) return it->second;
  auto kern = layout_cluster_kernel<IdT, kThreads>;
  int best = 8;  // portable cluster size
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxClusterCtas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kMaxClusterCtas;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0)
      best = kMaxClusterCtas;
  }
  cudaGetLastError();  // clear a refused query
  cache[{dev, smem}] = best;
  return best;
}

// One launch of the cluster kernel with CTAs of kThreads threads: up to 16
// CTAs of at least kSlotsPerClusterCta slots each (fewer for small
// batches), the CTA's ids staged in shared memory when they fit.
template <typename IdT, int kThreads>
cudaError_t launch_cluster_with(Params p, int n_ctas, cudaStream_t s, int *launches) {
  auto kern = layout_cluster_kernel<IdT, kThreads>;
  const int smem_max = max_dynamic_smem(reinterpret_cast<const void *>(kern));
  const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem_max);
  if (err != cudaSuccess) return err;
  constexpr int warps = kThreads / kWarp;
  if (n_ctas > 8)
    n_ctas = min(n_ctas, max_cluster_ctas<IdT, kThreads>(
                             cluster_smem_bytes(p.E, p.R, warps, kMaxClusterCtas, 0)));
  const long per_cta_slots = static_cast<long>((p.T + n_ctas - 1) / n_ctas) * p.k;
  int smem = cluster_smem_bytes(p.E, p.R, warps, n_ctas, 0);
  p.stage = 0;
  if (per_cta_slots <= kStageIdsMax) {
    const int staged = cluster_smem_bytes(p.E, p.R, warps, n_ctas, per_cta_slots);
    if (staged <= smem_max) {
      smem = staged;
      p.stage = 1;
    }
  }
  ++*launches;
  return launch_pdl(kern, dim3(n_ctas), dim3(kThreads), smem, s, n_ctas, p);
}

template <typename IdT>
cudaError_t launch_cluster(Params p, cudaStream_t s, int *launches) {
  const long N = static_cast<long>(p.T) * p.k;
  if (N <= kSmallSlots) return launch_cluster_with<IdT, kSmallThreads>(p, 1, s, launches);
  long want = (N + kSlotsPerClusterCta - 1) / kSlotsPerClusterCta;
  const int n_ctas = static_cast<int>(want < kMaxClusterCtas ? want : kMaxClusterCtas);
  // CTA size from the slots a CTA gets with the full cluster (a smaller
  // cluster only happens where 16 CTAs cannot run at once)
  const long per_cta_slots = static_cast<long>((p.T + n_ctas - 1) / n_ctas) * p.k;
  if (per_cta_slots <= kClusterSmallCtaSlots)
    return launch_cluster_with<IdT, kClusterThreadsSmall>(p, n_ctas, s, launches);
  return launch_cluster_with<IdT, kClusterThreads>(p, n_ctas, s, launches);
}

// The grid kernel: one CTA per SM, launched cooperatively (all CTAs
// resident at once, or the launch is refused) with programmatic stream
// serialization.  Returns the launch error; nothing runs when it fails.
template <typename IdT>
cudaError_t launch_grid(Params p, int ctas, void *ws, cudaStream_t s) {
  auto kern = layout_grid_kernel<IdT>;
  const long per_cta_slots = static_cast<long>((p.T + ctas - 1) / ctas) * p.k;
  const int smem_max = max_dynamic_smem(reinterpret_cast<const void *>(kern));
  int smem = grid_smem_bytes(p.E, p.R, 0);
  p.stage = 0;
  if (per_cta_slots <= kStageIdsMax && grid_smem_bytes(p.E, p.R, per_cta_slots) <= smem_max) {
    smem = grid_smem_bytes(p.E, p.R, per_cta_slots);
    p.stage = 1;
  }
  const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (err != cudaSuccess) return err;
  p.gbar = static_cast<unsigned *>(ws);
  // the testing switch of the bounded waits reaches the first barrier too
  p.first_polls = first_wait_polls() == 0 ? 0 : kMaxGridPolls;
  p.gcols = reinterpret_cast<int32_t *>(static_cast<char *>(ws) + kGridHeaderBytes);
  p.gtot = p.gcols + static_cast<long>(p.E + p.R) * ctas;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kGridThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

template <typename IdT>
cudaError_t launch_tiled(Params p, cudaStream_t s, int *launches) {
  const int C = p.E + p.R, ld = p.E + p.R + 1;
  const int count_smem = (kTileWarps * ld + C + (kTileThreads > C ? kTileThreads : C) + 1) *
                         static_cast<int>(sizeof(int));
  const int place_smem = (kTileWarps * ld + p.E + C) * static_cast<int>(sizeof(int));
  cudaError_t err =
      raise_dynamic_smem(reinterpret_cast<const void *>(layout_count_kernel<IdT>), count_smem);
  if (err != cudaSuccess) return err;
  err = raise_dynamic_smem(reinterpret_cast<const void *>(layout_place_kernel<IdT>), place_smem);
  if (err != cudaSuccess) return err;
  ++*launches;
  err = launch_pdl(layout_count_kernel<IdT>, dim3(p.ntiles), dim3(kTileThreads), count_smem, s,
                   1, p);
  if (err != cudaSuccess) return err;
  ++*launches;
  return launch_pdl(layout_place_kernel<IdT>, dim3(p.ntiles), dim3(kTileThreads), place_smem,
                    s, 1, p);
}

}  // namespace

size_t layout_workspace_bytes(int T, int k, int E, int R) {
  if (T <= 0) return 0;
  if (grid_path(T, k, E, R)) return grid_ws_bytes(E, R);
  if (cluster_path(T, k)) return 0;
  const int tile_T = tile_tokens(T);
  const long ntiles = (T + tile_T - 1) / tile_T;
  return kTicketBytes + static_cast<size_t>(ntiles) * (E + R) * sizeof(int32_t);
}

cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s, int *launches) {
  Params p{};
  p.idx = a.idx;
  p.T = a.T;
  p.k = a.k;
  p.E = a.E;
  p.R = a.R;
  const int G = a.E / a.R;
  p.g_magic = ((1ull << 32) + G - 1) / G;
  p.id_bits = 0;
  while ((1 << p.id_bits) < a.E) ++p.id_bits;
  p.cnt_e = a.cnt_e;
  p.cnt_r = a.cnt_r;
  p.off_e = a.off_e;
  p.off_r = a.off_r;
  p.slot_pos = a.slot_pos;
  p.recv_src = a.recv_src;
  p.in_rank = a.in_rank;
  p.d_err = a.d_err;
  if (a.ws != nullptr && grid_path(a.T, a.k, a.E, a.R)) {
    const int ctas = grid_ctas();
    cudaError_t err;
    if (a.id_kind == kIdsMask)
      err = launch_grid<uint8_t>(p, ctas, a.ws, s);
    else
      err = a.id_kind == kIdsInt64 ? launch_grid<int64_t>(p, ctas, a.ws, s)
                                   : launch_grid<int32_t>(p, ctas, a.ws, s);
    if (err == cudaSuccess) {
      ++*launches;
      return err;
    }
    // refused (for instance fewer SMs than CTAs in a green context): the
    // cluster kernel needs no co-residency beyond its own cluster
    cudaGetLastError();
  }
  if (cluster_path(a.T, a.k)) {
    if (a.id_kind == kIdsMask) return launch_cluster<uint8_t>(p, s, launches);
    return a.id_kind == kIdsInt64 ? launch_cluster<int64_t>(p, s, launches)
                                  : launch_cluster<int32_t>(p, s, launches);
  }
  p.tile_T = tile_tokens(a.T);
  p.ntiles = (a.T + p.tile_T - 1) / p.tile_T;
  p.ticket = static_cast<unsigned *>(a.ws);
  p.cols = reinterpret_cast<int32_t *>(static_cast<char *>(a.ws) + kTicketBytes);
  if (a.id_kind == kIdsMask) return launch_tiled<uint8_t>(p, s, launches);
  return a.id_kind == kIdsInt64 ? launch_tiled<int64_t>(p, s, launches)
                                : launch_tiled<int32_t>(p, s, launches);
}

}  // namespace ep
