// combine.cu -- gate-weighted sum of the expert outputs back into token
// order: out[t] = bf16(fma chain over slots j = 0..k-1 of w[t,j] * y[row]).
//
// Persistent grid-stride loop over work items (token t, chunk of its row).
// For each item a warp issues the loads of up to 8 slot rows at once
// (128-bit read-only streaming loads, so 8 x 16 B per lane are in flight),
// then folds them into fp32 accumulators strictly in slot order, and writes
// the chunk once with a coalesced streaming store.
#include <cuda_bf16.h>

#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kThreads = 256;
constexpr int kVec = 1;      // 16-byte vectors per lane per item
constexpr int kSlotBatch = 8;  // slot rows loaded together

__device__ __forceinline__ void fma_bf16x8(float *acc, float w, uint4 v) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = __fmaf_rn(w, __uint_as_float(in[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = __fmaf_rn(w, __uint_as_float(in[i] & 0xffff0000u), acc[2 * i + 1]);
  }
}

__device__ __forceinline__ uint4 to_bf16x8(const float *acc) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
    o[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int V>
__global__ void __launch_bounds__(kThreads, 2)
    combine_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                   const int32_t *__restrict__ slot_pos,
                   const float *__restrict__ w, uint4 *__restrict__ out,
                   long n_rows) {
  const int lane = threadIdx.x & 31;
  const int per_chunk = 32 * V;
  const int nchunks = (Hv + per_chunk - 1) / per_chunk;
  const long items = static_cast<long>(T) * nchunks;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long it = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int t = static_cast<int>(it / nchunks);
    const int c = static_cast<int>(it - static_cast<long>(t) * nchunks);
    const long tk = static_cast<long>(t) * k;
    const int sp = lane < k ? __ldg(slot_pos + tk + lane) : -1;
    const float wt = lane < k ? __ldg(w + tk + lane) : 0.0f;
    const int v0 = c * per_chunk + lane;

    float acc[V][8];
#pragma unroll
    for (int u = 0; u < V; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[u][e] = 0.0f;

    for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
      uint4 v[kSlotBatch][V];
      float wj[kSlotBatch];
      bool ok[kSlotBatch];
#pragma unroll
      for (int jj = 0; jj < kSlotBatch; ++jj) {
        const int j = j0 + jj;
        const int row = __shfl_sync(0xffffffffu, sp, j & 31);
        wj[jj] = __shfl_sync(0xffffffffu, wt, j & 31);
        ok[jj] = j < k && row >= 0 && row < n_rows;
        const uint4 *src = y + static_cast<long>(row) * Hv;
#pragma unroll
        for (int u = 0; u < V; ++u)
          v[jj][u] = ok[jj] && v0 + 32 * u < Hv ? ld_stream_v4(src + v0 + 32 * u)
                                                : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int jj = 0; jj < kSlotBatch; ++jj) {
        if (!ok[jj]) continue;  // a dropped slot adds nothing
#pragma unroll
        for (int u = 0; u < V; ++u) fma_bf16x8(acc[u], wj[jj], v[jj][u]);
      }
    }
    uint4 *dst = out + static_cast<long>(t) * Hv;
#pragma unroll
    for (int u = 0; u < V; ++u)
      if (v0 + 32 * u < Hv) st_stream_v4(dst + v0 + 32 * u, to_bf16x8(acc[u]));
  }
}

}  // namespace

cudaError_t launch_combine(const void *y, int T, int H, int k,
                           const int32_t *slot_pos, const float *w, void *out,
                           int num_sms, cudaStream_t s, int *launches) {
  const int Hv = H / 8;
  const long nchunks = (Hv + 32 * kVec - 1) / (32 * kVec);
  const long items = static_cast<long>(T) * nchunks;
  if (items == 0) return cudaSuccess;
  auto kern = combine_kernel<kVec>;
  const long grid = persistent_grid(reinterpret_cast<const void *>(kern), kThreads, items, num_sms);
  kern<<<grid, kThreads, 0, s>>>(static_cast<const uint4 *>(y), T, Hv, k, slot_pos, w,
                                 static_cast<uint4 *>(out), static_cast<long>(T) * k);
  ++*launches;
  return cudaGetLastError();
}

}  // namespace ep
