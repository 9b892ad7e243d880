// dispatch_bf16.cu -- token rows to expert-contiguous receive rows (bf16).
//
// A grid-stride loop over work items (token t, chunk c of its row), one
// warp per item.  A warp loads the chunk once with 128-bit read-only
// streaming loads, then writes it to each of the token's k receive rows
// with coalesced streaming stores, so HBM sees each source byte read once
// and each destination byte written once.  The slot rows of the token are
// fetched by lanes 0..k-1 and broadcast with shuffles.  Before waiting on
// the previous kernel, every warp asks L2 for the x chunks it will copy.
//
// On all SMs the grid holds one warp per item, so waves of CTAs follow one
// another as SMs free up (measured against a persistent grid of 8 CTAs per
// SM: 91 -> 84 us inside the prefill step); under an SM budget
// (num_sms > 0) the grid is persistent, sized to the budget.
#include <algorithm>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kThreads = 256;
constexpr int kBf16Vec = 2;  // 16-byte vectors per lane per item
// x bytes the kernel prefetches into L2 before its wait (half of the 126 MB
// L2: the whole token batch at the prefill shape; the first part of larger
// ones, which prefetching entirely slowed by 5 % as lines were evicted
// before their turn)
constexpr long kPrefetchBytes = 64L << 20;

// 8 CTAs per SM (at most 32 registers; the uncapped build took 36 and left
// room for 6): measured 0.7 us faster at the prefill shape.
template <int V>
__global__ void __launch_bounds__(kThreads, 8)
    dispatch_bf16_kernel(const uint4 *__restrict__ x, int T, int Hv, int k,
                         const int32_t *__restrict__ slot_pos,
                         uint4 *__restrict__ recv, long n_rows, long pf_warps) {
  const int lane = threadIdx.x & 31;
  const int per_chunk = 32 * V;
  const int nchunks = (Hv + per_chunk - 1) / per_chunk;
  const long items = static_cast<long>(T) * nchunks;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  {
    // ask L2 for x up front, one bulk prefetch per lane and item, before
    // waiting on the previous kernel (a prefetch only warms L2, which every
    // later write goes through, so it is safe even when that kernel writes
    // x).  The first pf_warps warps (those the SMs hold at once) take every
    // pf_warps-th item each, so that x streams into L2 in one burst while
    // the warps that copy it mostly write (prefill step 229.3-230.3 ->
    // 226.8-227.8 us against each warp prefetching only its own items).
    // Only the items of the first kPrefetchBytes of x in loop order: more
    // would be evicted before use.
    const long w0 = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long pf_end = w0 < pf_warps ? min(items, kPrefetchBytes / (per_chunk * 16)) : 0;
    for (long it = w0 + static_cast<long>(lane) * pf_warps; it < pf_end; it += 32 * pf_warps) {
      const int t = static_cast<int>(it / nchunks);
      const int c = static_cast<int>(it - static_cast<long>(t) * nchunks);
      prefetch_l2(x + static_cast<long>(t) * Hv + c * per_chunk,
                  min(per_chunk, Hv - c * per_chunk) * 16);
    }
  }
  pdl_wait();
  for (long it = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int t = static_cast<int>(it / nchunks);
    const int c = static_cast<int>(it - static_cast<long>(t) * nchunks);
    const int sp = lane < k ? __ldg(slot_pos + static_cast<long>(t) * k + lane) : -1;
    const int v0 = c * per_chunk + lane;
    const uint4 *src = x + static_cast<long>(t) * Hv;
    uint4 v[V];
#pragma unroll
    for (int u = 0; u < V; ++u)
      v[u] = v0 + 32 * u < Hv ? ld_stream_v4(src + v0 + 32 * u) : make_uint4(0, 0, 0, 0);
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xffffffffu, sp, j);
      if (row < 0 || row >= n_rows) continue;  // uniform across the warp
      uint4 *dst = recv + static_cast<long>(row) * Hv;
#pragma unroll
      for (int u = 0; u < V; ++u)
        if (v0 + 32 * u < Hv) st_stream_v4(dst + v0 + 32 * u, v[u]);
    }
  }
}

}  // namespace

cudaError_t launch_dispatch_bf16(const void *x, int T, int H, int k,
                                 const int32_t *slot_pos, void *recv, long n_rows,
                                 int num_sms, int32_t * /*d_err*/, cudaStream_t s,
                                 int *launches) {
  const int Hv = H / 8;
  const long nchunks = (Hv + 32 * kBf16Vec - 1) / (32 * kBf16Vec);
  const long items = static_cast<long>(T) * nchunks;
  if (items == 0) return cudaSuccess;
  auto kern = dispatch_bf16_kernel<kBf16Vec>;
  constexpr long kWarpsPerCta = kThreads / 32;
  constexpr long kMaxGridX = 2147483647;
  const long grid =
      num_sms > 0
          ? persistent_grid(reinterpret_cast<const void *>(kern), kThreads, 0, items, num_sms)
          : std::min((items + kWarpsPerCta - 1) / kWarpsPerCta, kMaxGridX);
  // warps resident at once: every SM's 64 warp slots, or the whole grid
  const int sms = num_sms > 0 ? num_sms : device_sm_count();
  const long pf_warps = std::min(grid * kWarpsPerCta, static_cast<long>(sms) * 64);
  ++*launches;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), 0, s, 1, static_cast<const uint4 *>(x), T,
                    Hv, k, slot_pos, static_cast<uint4 *>(recv), n_rows, pf_warps);
}

}  // namespace ep
