// layout.cu -- the dispatch layout on the GPU: per-expert and per-rank
// counts, the token-in-rank mask, exclusive prefix offsets and the stable
// receive row of every (token, slot).
//
// Two paths, both deterministic (no ordering ever depends on atomics) and
// neither with a CTA that waits on another through memory:
//  * cluster (T*k <= kClusterMaxSlots): one launch of a thread-block
//    cluster of up to 16 CTAs (1 CTA for small batches such as a 128-token
//    decode step).  Each CTA counts its contiguous token range, the CTAs
//    exchange their per-expert counts through distributed shared memory
//    between two hardware cluster barriers, and every CTA then places its
//    own slots.  No global workspace.
//  * tiled (larger batches): a counting kernel writes one histogram row per
//    tile of tokens to the caller's workspace, and the last tile to finish
//    (ticket taken with atomicInc, which wraps it back to 0) turns the rows
//    into absolute per-tile bases and the global offsets; a placing kernel
//    then gives every slot its row.
// Inside a CTA each warp owns a contiguous run of slots.  Stable ranks
// within 32 slots come from __match_any_sync + popc of the lower lanes; the
// per-warp running bases come from per-warp histograms scanned across warps,
// so slot order = token-major order exactly.
#include <cooperative_groups.h>

#include <map>
#include <mutex>

#include "ep_internal.cuh"

namespace ep {
namespace {

namespace cg = cooperative_groups;

constexpr int kClusterThreads = 1024;
constexpr int kClusterWarps = kClusterThreads / kWarp;
constexpr int kMaxClusterCtas = 16;
constexpr long kClusterMaxSlots = 1L << 19;
constexpr long kSlotsPerClusterCta = 4096;  // below this, fewer CTAs

constexpr int kTileThreads = 512;
constexpr int kTileWarps = kTileThreads / kWarp;
constexpr int kTileTokensMin = 128;
constexpr int kMaxTiles = 296;  // 2 per SM on a 148-SM B200
constexpr int kTicketBytes = 16;

struct Params {
  const void *idx;
  int T, k, E, R, G;
  int32_t *cnt_e, *cnt_r, *off_e, *off_r, *slot_pos, *recv_src;
  uint8_t *in_rank;
  int32_t *d_err;
  unsigned *ticket;  // tiled path
  int32_t *cols;     // tiled path: [ntiles][E + R]
  int tile_T, ntiles;
};

// Expert id from a raw id value: -1 for a dropped or bad slot (a bad one
// is reported through d_err when given).
__device__ __forceinline__ int check_id(long long e, int E, int32_t *d_err) {
  if (e >= 0 && e < E) return static_cast<int>(e);
  if (e != -1 && d_err != nullptr) atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_INDEX);
  return -1;
}

// Ids are read kIdBatch at a time per lane, all loads issued before any is
// used, so a warp pays one memory round trip per kIdBatch * 32 slots.
constexpr int kIdBatch = 8;

template <typename IdT>
__device__ __forceinline__ void load_id_batch(const IdT *idx, long c0, long end,
                                              long long (&v)[kIdBatch]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int b = 0; b < kIdBatch; ++b) {
    const long i = c0 + 32 * b + lane;
    v[b] = i < end ? static_cast<long long>(idx[i]) : -1;
  }
}

// In-place exclusive scan of a[0..n) in shared memory by the whole block;
// returns the total.  warp_tmp: 32 ints of shared memory.
__device__ int block_exclusive_scan(int *a, int n, int *warp_tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, wid = tid >> 5, nw = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  int local = 0;
  for (int i = beg; i < end; ++i) local += a[i];
  int v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tmp[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int t = lane < nw ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    if (lane < nw) warp_tmp[lane] = t;
  }
  __syncthreads();
  int run = v - local + (wid > 0 ? warp_tmp[wid - 1] : 0);
  const int total = warp_tmp[nw - 1];
  for (int i = beg; i < end; ++i) {
    const int c = a[i];
    a[i] = run;
    run += c;
  }
  __syncthreads();
  return total;
}

// Contiguous, 32-aligned slice [b, *end) of [0, n) for warp w of nw.
__device__ __forceinline__ long warp_slice(long n, int w, int nw, long *end) {
  const long s = ((n + nw - 1) / nw + 31) / 32 * 32;
  const long b = min(n, s * w);
  *end = min(n, b + s);
  return b;
}

// Per-warp counts of the kept ids in slots [beg, end) (warp-uniform range).
template <typename IdT>
__device__ void count_segment(const IdT *idx, long beg, long end, int E, int32_t *d_err,
                              int *hist_w) {
  for (long c0 = beg; c0 < end; c0 += 32 * kIdBatch) {
    long long v[kIdBatch];
    load_id_batch(idx, c0, end, v);
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int e = check_id(v[b], E, d_err);
      if (e >= 0) atomicAdd(&hist_w[e], 1);
    }
  }
}

// Gives each slot in [beg, end) its row; base[e] holds the next free row of
// expert e for this warp and is advanced as slots are placed.
template <typename IdT>
__device__ void place_segment(const IdT *idx, long beg, long end, int k, int E, int *base,
                              int32_t *slot_pos, int32_t *recv_src) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  for (long c0 = beg; c0 < end; c0 += 32 * kIdBatch) {
    long long v[kIdBatch];
    load_id_batch(idx, c0, end, v);
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      if (c0 + 32 * b >= end) break;  // uniform across the warp
      const long i = c0 + 32 * b + lane;
      const int e = check_id(v[b], E, nullptr);
      // lanes without a kept slot get keys no other lane can share
      const int key = e >= 0 ? e : -2 - lane;
      const unsigned peers = __match_any_sync(0xffffffffu, key);
      int pos = -1;
      if (e >= 0) {
        pos = base[e] + __popc(peers & lt);
        recv_src[pos] = static_cast<int32_t>(i / k);
      }
      if (i < end) slot_pos[i] = pos;
      __syncwarp();
      if (e >= 0 && (peers & lt) == 0) base[e] += __popc(peers);
      __syncwarp();
    }
  }
}

// Token-in-rank mask rows for tokens [t_beg, t_end) and their per-rank
// counts (atomics into rank_cnt[R]: counts only, no order involved).
template <typename IdT>
__device__ void rank_mask(const Params &p, int t_beg, int t_end, int *rank_cnt) {
  const IdT *idx = static_cast<const IdT *>(p.idx);
  for (int t = t_beg + threadIdx.x; t < t_end; t += blockDim.x) {
    const long base = static_cast<long>(t) * p.k;
    unsigned long long m = 0;
    for (int j0 = 0; j0 < p.k; j0 += kIdBatch) {
      long long v[kIdBatch];
#pragma unroll
      for (int b = 0; b < kIdBatch; ++b)
        v[b] = j0 + b < p.k ? static_cast<long long>(idx[base + j0 + b]) : -1;
#pragma unroll
      for (int b = 0; b < kIdBatch; ++b) {
        const int e = check_id(v[b], p.E, nullptr);
        if (e >= 0) m |= 1ull << (e / p.G);
      }
    }
    uint8_t *row = p.in_rank + static_cast<long>(t) * p.R;
    for (int r = 0; r < p.R; ++r) row[r] = static_cast<uint8_t>((m >> r) & 1u);
    while (m) {
      const int r = __ffsll(static_cast<long long>(m)) - 1;
      atomicAdd(&rank_cnt[r], 1);
      m &= m - 1;
    }
  }
}

// ------------------------------------------------------------- cluster path

int cluster_smem_bytes(int E, int R) {
  return (kClusterWarps * E + 3 * (E + R) + 32) * static_cast<int>(sizeof(int));
}

template <typename IdT>
__global__ void __launch_bounds__(kClusterThreads, 1) layout_cluster_kernel(Params p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int n_ctas = static_cast<int>(cluster.num_blocks());
  const int rank = static_cast<int>(cluster.block_rank());
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R;
  int *hist = smem;                       // [warps][E]
  int *mine = hist + kClusterWarps * E;   // [C] this CTA's counts, read by all CTAs
  int *before = mine + C;                 // [C] counts of the lower-ranked CTAs
  int *tot = before + C;                  // [C] totals, then exclusive offsets
  int *warp_tmp = tot + C;                // [32]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tid = threadIdx.x, nt = blockDim.x, w = tid >> 5;

  const int per_cta = (p.T + n_ctas - 1) / n_ctas;
  const int t_beg = min(p.T, rank * per_cta);
  const int t_end = min(p.T, t_beg + per_cta);
  const long s_beg = static_cast<long>(t_beg) * p.k;
  const long n = static_cast<long>(t_end - t_beg) * p.k;

  for (int i = tid; i < kClusterWarps * E + C; i += nt) smem[i] = 0;
  __syncthreads();
  long seg_end;
  const long seg_beg = warp_slice(n, w, kClusterWarps, &seg_end);
  count_segment(idx, s_beg + seg_beg, s_beg + seg_end, E, p.d_err, hist + w * E);
  rank_mask<IdT>(p, t_beg, t_end, mine + E);
  __syncthreads();
  // hist[w][e] -> count of the earlier warps; mine[e] -> this CTA's total
  for (int e = tid; e < E; e += nt) {
    int run = 0;
    for (int v = 0; v < kClusterWarps; ++v) {
      const int c = hist[v * E + e];
      hist[v * E + e] = run;
      run += c;
    }
    mine[e] = run;
  }
  cluster.sync();  // every CTA's `mine` is complete and visible
  for (int c = tid; c < C; c += nt) {
    int b = 0, a = 0;
    for (int r = 0; r < n_ctas; ++r) {
      const int v = cluster.map_shared_rank(mine, r)[c];
      b += r < rank ? v : 0;
      a += v;
    }
    before[c] = b;
    tot[c] = a;
  }
  cluster.sync();  // no CTA reads another's shared memory after this
  if (rank == 0)
    for (int c = tid; c < C; c += nt) {
      if (c < E) p.cnt_e[c] = tot[c];
      else p.cnt_r[c - E] = tot[c];
    }
  __syncthreads();
  const int n_kept = block_exclusive_scan(tot, E, warp_tmp);
  const int n_tok = block_exclusive_scan(tot + E, R, warp_tmp);
  if (rank == 0) {
    for (int c = tid; c < C; c += nt) {
      if (c < E) p.off_e[c] = tot[c];
      else p.off_r[c - E] = tot[c];
    }
    if (tid == 0) {
      p.off_e[E] = n_kept;
      p.off_r[R] = n_tok;
    }
  }
  for (int e = tid; e < E; e += nt) {
    const int b = tot[e] + before[e];
    for (int v = 0; v < kClusterWarps; ++v) hist[v * E + e] += b;
  }
  __syncthreads();
  place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * E, p.slot_pos,
                p.recv_src);
  const long N = static_cast<long>(p.T) * p.k;
  for (long r = n_kept + static_cast<long>(rank) * nt + tid; r < N;
       r += static_cast<long>(n_ctas) * nt)
    p.recv_src[r] = -1;
}

// ------------------------------------------------------------- tiled path

template <typename IdT>
__global__ void __launch_bounds__(kTileThreads) layout_count_kernel(Params p) {
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R;
  const int tid = threadIdx.x, nt = blockDim.x;
  int *col = smem;                    // [C]   this tile's counts, later totals
  int *part = col + C;                // [max(nt, C)] partial column sums
  int *warp_tmp = part + max(nt, C);  // [32]
  int *flag = warp_tmp + 32;          // [1]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tile = blockIdx.x;
  const int t_beg = tile * p.tile_T;
  const int t_end = min(p.T, t_beg + p.tile_T);

  for (int i = tid; i < C; i += nt) col[i] = 0;
  __syncthreads();
  const long s_end = static_cast<long>(t_end) * p.k;
  for (long c0 = static_cast<long>(t_beg) * p.k; c0 < s_end; c0 += static_cast<long>(nt) * kIdBatch) {
    long long v[kIdBatch];
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const long i = c0 + static_cast<long>(b) * nt + tid;
      v[b] = i < s_end ? static_cast<long long>(idx[i]) : -1;
    }
#pragma unroll
    for (int b = 0; b < kIdBatch; ++b) {
      const int e = check_id(v[b], E, p.d_err);
      if (e >= 0) atomicAdd(&col[e], 1);
    }
  }
  rank_mask<IdT>(p, t_beg, t_end, col + E);
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
    else p.cnt_r[c - E] = s;
  }
  __syncthreads();
  const int n_kept = block_exclusive_scan(col, E, warp_tmp);
  const int n_tok = block_exclusive_scan(col + E, R, warp_tmp);
  for (int c = tid; c < C; c += nt) {
    if (c < E) p.off_e[c] = col[c];
    else p.off_r[c - E] = col[c];
  }
  if (tid == 0) {
    p.off_e[E] = n_kept;
    p.off_r[R] = n_tok;
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
  extern __shared__ int smem[];
  const int E = p.E, C = p.E + p.R;
  int *hist = smem;  // [warps][E]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tid = threadIdx.x, w = tid >> 5;
  const int tile = blockIdx.x;
  const int t_beg = tile * p.tile_T;
  const int t_end = min(p.T, t_beg + p.tile_T);
  const long s_beg = static_cast<long>(t_beg) * p.k;
  const long n = static_cast<long>(t_end - t_beg) * p.k;

  for (int i = tid; i < kTileWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  long seg_end;
  const long seg_beg = warp_slice(n, w, kTileWarps, &seg_end);
  count_segment(idx, s_beg + seg_beg, s_beg + seg_end, E, nullptr, hist + w * E);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = __ldcg(&p.cols[static_cast<long>(tile) * C + e]);
    for (int v = 0; v < kTileWarps; ++v) {
      const int c = hist[v * E + e];
      hist[v * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * E, p.slot_pos,
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

// Largest cluster (<= 16 CTAs) the device can schedule for this kernel with
// `smem` bytes per CTA; cached per (device, id type, smem size).
template <typename IdT>
int max_cluster_ctas(int smem) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, smem});
  if (it != cache.end()) return it->second;
  auto kern = layout_cluster_kernel<IdT>;
  int best = 8;  // portable cluster size
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxClusterCtas);
    cfg.blockDim = dim3(kClusterThreads);
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

template <typename IdT>
cudaError_t launch_cluster(Params p, cudaStream_t s, int *launches) {
  auto kern = layout_cluster_kernel<IdT>;
  const int smem = cluster_smem_bytes(p.E, p.R);
  cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
  if (err != cudaSuccess) return err;
  const long N = static_cast<long>(p.T) * p.k;
  long want = (N + kSlotsPerClusterCta - 1) / kSlotsPerClusterCta;
  if (want < 1) want = 1;
  const int cap = want > 8 ? max_cluster_ctas<IdT>(smem) : 8;
  const int n_ctas = static_cast<int>(want < cap ? want : cap);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_ctas);
  cfg.blockDim = dim3(kClusterThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = n_ctas;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  err = cudaLaunchKernelEx(&cfg, kern, p);
  ++*launches;
  return err;
}

template <typename IdT>
cudaError_t launch_tiled(Params p, cudaStream_t s, int *launches) {
  const int C = p.E + p.R;
  const int count_smem =
      (C + (kTileThreads > C ? kTileThreads : C) + 32 + 1) * static_cast<int>(sizeof(int));
  const int place_smem = kTileWarps * p.E * static_cast<int>(sizeof(int));
  cudaError_t err =
      raise_dynamic_smem(reinterpret_cast<const void *>(layout_place_kernel<IdT>), place_smem);
  if (err != cudaSuccess) return err;
  layout_count_kernel<IdT><<<p.ntiles, kTileThreads, count_smem, s>>>(p);
  ++*launches;
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  layout_place_kernel<IdT><<<p.ntiles, kTileThreads, place_smem, s>>>(p);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t layout_workspace_bytes(int T, int k, int E, int R) {
  if (T <= 0 || cluster_path(T, k)) return 0;
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
  p.G = a.E / a.R;
  p.cnt_e = a.cnt_e;
  p.cnt_r = a.cnt_r;
  p.off_e = a.off_e;
  p.off_r = a.off_r;
  p.slot_pos = a.slot_pos;
  p.recv_src = a.recv_src;
  p.in_rank = a.in_rank;
  p.d_err = a.d_err;
  if (cluster_path(a.T, a.k))
    return a.idx_is_int64 ? launch_cluster<int64_t>(p, s, launches)
                          : launch_cluster<int32_t>(p, s, launches);
  p.tile_T = tile_tokens(a.T);
  p.ntiles = (a.T + p.tile_T - 1) / p.tile_T;
  p.ticket = static_cast<unsigned *>(a.ws);
  p.cols = reinterpret_cast<int32_t *>(static_cast<char *>(a.ws) + kTicketBytes);
  return a.idx_is_int64 ? launch_tiled<int64_t>(p, s, launches)
                        : launch_tiled<int32_t>(p, s, launches);
}

}  // namespace ep
