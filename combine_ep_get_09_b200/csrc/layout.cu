// layout.cu -- the dispatch layout on the GPU: per-expert and per-rank
// counts, the token-in-rank mask, exclusive prefix offsets and the stable
// receive row of every (token, slot).
//
// Two paths, both deterministic (no ordering ever depends on atomics):
//  * single block (T*k <= kSingleMaxSlots, e.g. a 128-token decode batch):
//    one launch of 512 threads;
//  * tiled (larger batches): a counting kernel writes one histogram row per
//    tile of tokens, and the last tile to finish (ticket taken with
//    atomicInc, so it resets itself) turns the rows into absolute per-tile
//    bases and the global offsets; a placing kernel then gives every slot
//    its row.
// Inside a block each warp owns a contiguous run of slots.  Stable ranks
// within 32 slots come from __match_any_sync + popc of the lower lanes; the
// per-warp running bases are built from per-warp histograms scanned across
// warps, so slot order = token-major order exactly.
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kLayoutThreads = 512;
constexpr int kLayoutWarps = kLayoutThreads / kWarp;
constexpr int kSingleMaxSlots = 16384;
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

// Expert id of flat slot i, or -1 for a dropped or bad slot (a bad one is
// reported through d_err when given).
template <typename IdT>
__device__ __forceinline__ int load_id(const IdT *idx, long i, int E,
                                       int32_t *d_err) {
  const long long e = static_cast<long long>(idx[i]);
  if (e >= 0 && e < E) return static_cast<int>(e);
  if (e != -1 && d_err != nullptr)
    atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_INDEX);
  return -1;
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

// Per-warp counts of the kept ids in slots [beg, end) (warp-uniform range).
template <typename IdT>
__device__ void count_segment(const IdT *idx, long beg, long end, int E,
                              int32_t *d_err, int *hist_w) {
  const int lane = threadIdx.x & 31;
  for (long c0 = beg; c0 < end; c0 += 32) {
    const long i = c0 + lane;
    const int e = i < end ? load_id(idx, i, E, d_err) : -1;
    if (e >= 0) atomicAdd(&hist_w[e], 1);
  }
}

// Gives each slot in [beg, end) its row; base[e] holds the next free row of
// expert e for this warp and is advanced as slots are placed.
template <typename IdT>
__device__ void place_segment(const IdT *idx, long beg, long end, int k,
                              int E, int *base, int32_t *slot_pos,
                              int32_t *recv_src) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = lanemask_lt();
  for (long c0 = beg; c0 < end; c0 += 32) {
    const long i = c0 + lane;
    const bool in = i < end;
    const int e = in ? load_id(idx, i, E, nullptr) : -1;
    // lanes without a kept slot get keys no other lane can share
    const int key = e >= 0 ? e : -2 - lane;
    const unsigned peers = __match_any_sync(0xffffffffu, key);
    int pos = -1;
    if (e >= 0) {
      pos = base[e] + __popc(peers & lt);
      recv_src[pos] = static_cast<int32_t>(i / k);
    }
    if (in) slot_pos[i] = pos;
    __syncwarp();
    if (e >= 0 && (peers & lt) == 0) base[e] += __popc(peers);
    __syncwarp();
  }
}

// Token-in-rank mask rows for tokens [t_beg, t_end) and their per-rank
// counts (atomics into rank_cnt[R]: counts only, no order involved).
template <typename IdT>
__device__ void rank_mask(const Params &p, int t_beg, int t_end,
                          int *rank_cnt) {
  const IdT *idx = static_cast<const IdT *>(p.idx);
  for (int t = t_beg + threadIdx.x; t < t_end; t += blockDim.x) {
    unsigned long long m = 0;
    for (int j = 0; j < p.k; ++j) {
      const int e = load_id(idx, static_cast<long>(t) * p.k + j, p.E, nullptr);
      if (e >= 0) m |= 1ull << (e / p.G);
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

__device__ __forceinline__ long warp_slice(long n, int w, long *end) {
  // contiguous, 32-aligned slices of [0, n) for the block's warps
  const long s = ((n + kLayoutWarps - 1) / kLayoutWarps + 31) / 32 * 32;
  const long b = min(n, s * w);
  *end = min(n, b + s);
  return b;
}

// ------------------------------------------------------- single-block path

template <typename IdT>
__global__ void __launch_bounds__(kLayoutThreads)
    layout_single_kernel(Params p) {
  extern __shared__ int smem[];
  const int E = p.E, R = p.R;
  int *hist = smem;                         // [warps][E]
  int *tot = hist + kLayoutWarps * E;       // [E]
  int *rcnt = tot + E;                      // [R]
  int *warp_tmp = rcnt + R;                 // [32]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const long N = static_cast<long>(p.T) * p.k;
  const int tid = threadIdx.x, w = tid >> 5;

  for (int i = tid; i < kLayoutWarps * E + E + R; i += blockDim.x) smem[i] = 0;
  __syncthreads();

  long seg_end;
  const long seg_beg = warp_slice(N, w, &seg_end);
  count_segment(idx, seg_beg, seg_end, E, p.d_err, hist + w * E);
  rank_mask<IdT>(p, 0, p.T, rcnt);
  __syncthreads();

  // per-expert totals; hist[w][e] -> count of earlier warps
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int v = 0; v < kLayoutWarps; ++v) {
      const int c = hist[v * E + e];
      hist[v * E + e] = run;
      run += c;
    }
    tot[e] = run;
    p.cnt_e[e] = run;
  }
  for (int r = tid; r < R; r += blockDim.x) p.cnt_r[r] = rcnt[r];
  __syncthreads();
  const int n_kept = block_exclusive_scan(tot, E, warp_tmp);
  const int n_tok = block_exclusive_scan(rcnt, R, warp_tmp);
  for (int e = tid; e < E; e += blockDim.x) {
    p.off_e[e] = tot[e];
    for (int v = 0; v < kLayoutWarps; ++v) hist[v * E + e] += tot[e];
  }
  for (int r = tid; r < R; r += blockDim.x) p.off_r[r] = rcnt[r];
  if (tid == 0) {
    p.off_e[E] = n_kept;
    p.off_r[R] = n_tok;
  }
  __syncthreads();

  place_segment(idx, seg_beg, seg_end, p.k, E, hist + w * E, p.slot_pos,
                p.recv_src);
  for (long r = n_kept + tid; r < N; r += blockDim.x) p.recv_src[r] = -1;
}

// -------------------------------------------------------------- tiled path

template <typename IdT>
__global__ void __launch_bounds__(kLayoutThreads)
    layout_count_kernel(Params p) {
  extern __shared__ int smem[];
  const int E = p.E, R = p.R, C = E + R;
  const int tid = threadIdx.x, nt = blockDim.x;
  int *col = smem;                 // [C]   this tile's counts, later totals
  int *part = col + C;             // [max(nt, C)] partial column sums
  int *warp_tmp = part + max(nt, C);  // [32]
  int *flag = warp_tmp + 32;       // [1]
  const IdT *idx = static_cast<const IdT *>(p.idx);
  const int tile = blockIdx.x;
  const int t_beg = tile * p.tile_T;
  const int t_end = min(p.T, t_beg + p.tile_T);

  for (int i = tid; i < C; i += nt) col[i] = 0;
  __syncthreads();
  const long s_end = static_cast<long>(t_end) * p.k;
  for (long i = static_cast<long>(t_beg) * p.k + tid; i < s_end; i += nt) {
    const int e = load_id(idx, i, E, p.d_err);
    if (e >= 0) atomicAdd(&col[e], 1);
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

  // column totals, each column split into P contiguous runs of tiles
  const int P = max(1, nt / C);
  const int chunk = (p.ntiles + P - 1) / P;
  for (int q = tid; q < C * P; q += nt) {
    const int c = q % C, pp = q / C;
    const int b = pp * chunk, e_ = min(p.ntiles, b + chunk);
    int s = 0;
#pragma unroll 8
    for (int tl = b; tl < e_; ++tl) s += __ldcg(&p.cols[static_cast<long>(tl) * C + c]);
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
    for (int tl = b; tl < e_; ++tl) {
      int32_t *cell = &p.cols[static_cast<long>(tl) * C + c];
      const int v = __ldcg(cell);
      *cell = base;
      base += v;
    }
  }
}

template <typename IdT>
__global__ void __launch_bounds__(kLayoutThreads)
    layout_place_kernel(Params p) {
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

  for (int i = tid; i < kLayoutWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  long seg_end;
  const long seg_beg = warp_slice(n, w, &seg_end);
  count_segment(idx, s_beg + seg_beg, s_beg + seg_end, E, nullptr, hist + w * E);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) {
    int run = __ldcg(&p.cols[static_cast<long>(tile) * C + e]);
    for (int v = 0; v < kLayoutWarps; ++v) {
      const int c = hist[v * E + e];
      hist[v * E + e] = run;
      run += c;
    }
  }
  __syncthreads();
  place_segment(idx, s_beg + seg_beg, s_beg + seg_end, p.k, E, hist + w * E,
                p.slot_pos, p.recv_src);

  // rows nobody fills
  const long N = static_cast<long>(p.T) * p.k;
  const long n_kept = __ldcg(&p.off_e[E]);
  for (long r = n_kept + static_cast<long>(blockIdx.x) * blockDim.x + tid; r < N;
       r += static_cast<long>(gridDim.x) * blockDim.x)
    p.recv_src[r] = -1;
}

int tile_tokens(int T) {
  const int t = (T + kMaxTiles - 1) / kMaxTiles;
  return t > kTileTokensMin ? t : kTileTokensMin;
}

bool single_path(int T, int k) {
  return static_cast<long>(T) * k <= kSingleMaxSlots;
}

// Dynamic shared memory caps, sized for EP_MAX_E / EP_MAX_R and set once per
// device and kernel.
constexpr int kSingleSmemCap =
    (kLayoutWarps * EP_MAX_E + EP_MAX_E + EP_MAX_R + 32) * sizeof(int);
constexpr int kPlaceSmemCap = kLayoutWarps * EP_MAX_E * sizeof(int);
constexpr int kMaxDevices = 64;

template <typename IdT>
cudaError_t raise_smem_caps() {
  static bool done[kMaxDevices] = {};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < kMaxDevices && done[dev]) return cudaSuccess;
  err = cudaFuncSetAttribute(layout_single_kernel<IdT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSingleSmemCap);
  if (err == cudaSuccess)
    err = cudaFuncSetAttribute(layout_place_kernel<IdT>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kPlaceSmemCap);
  if (err == cudaSuccess && dev < kMaxDevices) done[dev] = true;
  return err;
}

template <typename IdT>
cudaError_t launch_typed(Params p, cudaStream_t s, int *launches) {
  cudaError_t err = raise_smem_caps<IdT>();
  if (err != cudaSuccess) return err;
  if (single_path(p.T, p.k)) {
    const int smem = (kLayoutWarps * p.E + p.E + p.R + 32) * sizeof(int);
    layout_single_kernel<IdT><<<1, kLayoutThreads, smem, s>>>(p);
    ++*launches;
    return cudaGetLastError();
  }
  const int C = p.E + p.R;
  const int count_smem =
      (C + (kLayoutThreads > C ? kLayoutThreads : C) + 32 + 1) * sizeof(int);
  const int place_smem = kLayoutWarps * p.E * sizeof(int);
  layout_count_kernel<IdT><<<p.ntiles, kLayoutThreads, count_smem, s>>>(p);
  ++*launches;
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  layout_place_kernel<IdT><<<p.ntiles, kLayoutThreads, place_smem, s>>>(p);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace

size_t layout_workspace_bytes(int T, int k, int E, int R) {
  if (T <= 0 || single_path(T, k)) return 0;
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
  if (!single_path(a.T, a.k)) {
    p.tile_T = tile_tokens(a.T);
    p.ntiles = (a.T + p.tile_T - 1) / p.tile_T;
    p.ticket = static_cast<unsigned *>(a.ws);
    p.cols = reinterpret_cast<int32_t *>(static_cast<char *>(a.ws) + kTicketBytes);
  }
  return a.idx_is_int64 ? launch_typed<int64_t>(p, s, launches)
                        : launch_typed<int32_t>(p, s, launches);
}

}  // namespace ep
