// combine.cu -- gate-weighted sum of the expert outputs back into token
// order: out[t] = bf16(fma chain over slots j = 0..k-1 of w[t,j] * y[row]),
// every w[t,j] = 1 when no weights are given (a plain sum, as combining
// per-rank partial outputs needs).
//
// Two kernels, both fp32 fma chains in slot order (so both bit-identical):
//
//  * combine_bulk_kernel (k <= 8, the common case): a bulk-copy (TMA)
//    pipeline.  A CTA of kChunkVec threads walks a contiguous range of
//    work items (token t, chunk c of kChunkVec 16-byte vectors).  Thread 0
//    gathers the chunk of each of the token's k slot rows into shared
//    memory with cp.async.bulk (one copy per row, completing on the stage's
//    mbarrier), kStages items ahead; every thread then folds its 16 bytes
//    of the k rows and writes one 16-byte vector of the output.  The bytes
//    in flight live in shared memory, not registers, which is what keeps
//    HBM busy on this read-dominated gather.
//  * combine_reg_kernel (any k <= 32): a warp per item with 128-bit loads
//    of 8 slot rows at a time into registers.
#include <cuda_bf16.h>

#include "bulk.cuh"
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kRegThreads = 256;
constexpr int kSlotBatch = 8;    // slot rows loaded together (register path)
constexpr int kBulkMaxK = 8;     // slot rows one bulk stage holds
constexpr int kChunkVec = 256;   // 16-byte vectors per row chunk = threads
constexpr int kStages = 2;       // items in flight per CTA
constexpr int kBulkSmem = kStages * kBulkMaxK * kChunkVec * 16;

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

__global__ void __launch_bounds__(kChunkVec)
    combine_bulk_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                        const int32_t *__restrict__ slot_pos, const float *__restrict__ w,
                        uint4 *__restrict__ out, long n_rows, int32_t *d_err) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  uint4 *stage_buf = reinterpret_cast<uint4 *>(smem_raw);  // [kStages][kBulkMaxK][kChunkVec]
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int stage_row[kStages][kBulkMaxK];
  __shared__ float stage_w[kStages][kBulkMaxK];

  const int tid = threadIdx.x, lane = tid & 31;
  const int nchunks = (Hv + kChunkVec - 1) / kChunkVec;
  const long items = static_cast<long>(T) * nchunks;
  // CTA b walks items [items * b / grid, items * (b + 1) / grid): the
  // shares differ by at most one item
  const long first = items * blockIdx.x / gridDim.x;
  const long n_mine = items * (blockIdx.x + 1) / gridDim.x - first;

  pdl_trigger();
  if (tid == 0) {
    // every lane of warp 0 arrives once per phase (see issue)
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], kWarp);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();

  // warp 0: lane j < k gathers the chunk of item i's slot row j into stage
  // i % kStages.  Each lane announces its own bytes with its arrival, so
  // the row indices and weights it leaves in shared memory are published
  // with it; dropped slots arrive with 0 bytes.
  auto issue = [&](long i) {
    const long it = first + i;
    const int s = static_cast<int>(i % kStages);
    const int t = static_cast<int>(it / nchunks);
    const int v0 = static_cast<int>(it % nchunks) * kChunkVec;
    const unsigned bytes = static_cast<unsigned>(min(kChunkVec, Hv - v0)) * 16u;
    int r = -1;
    if (lane < k) {
      r = __ldg(slot_pos + static_cast<long>(t) * k + lane);
      const float wj = w != nullptr ? __ldg(w + static_cast<long>(t) * k + lane) : 1.0f;
      if (r < 0 || r >= n_rows) r = -1;
      stage_row[s][lane] = r;
      stage_w[s][lane] = wj;
    } else if (lane < kBulkMaxK) {
      stage_row[s][lane] = -1;
    }
    mbar_arrive_expect_tx(&full[s], r >= 0 ? bytes : 0u);
    if (r >= 0)
      bulk_load(stage_buf + (s * kBulkMaxK + lane) * kChunkVec, y + static_cast<long>(r) * Hv + v0,
                bytes, &full[s]);
  };

  if (tid < kWarp)
    for (long i = 0; i < min(static_cast<long>(kStages), n_mine); ++i) issue(i);

  long i = 0;
  bool timed_out = false;
  for (; i < n_mine; ++i) {
    const int s = static_cast<int>(i % kStages);
    const long it = first + i;
    const int t = static_cast<int>(it / nchunks);
    const int v0 = static_cast<int>(it % nchunks) * kChunkVec;
    const bool ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kStages) & 1));
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    if (tid < Hv - v0) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int j = 0; j < kBulkMaxK; ++j)
        if (stage_row[s][j] >= 0)  // dropped slots add nothing
          fma_bf16x8(acc, stage_w[s][j], stage_buf[(s * kBulkMaxK + j) * kChunkVec + tid]);
      st_stream_v4(out + static_cast<long>(t) * Hv + v0 + tid, to_bf16x8(acc));
    }
    __syncthreads();  // stage s fully read
    if (tid < kWarp && i + kStages < n_mine) issue(i + kStages);
  }
  if (timed_out && tid == 0) {
    if (d_err != nullptr) atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_TIMEOUT);
    // let the copies still in flight land before the CTA's memory goes away
    for (long q = i; q < min(n_mine, i + kStages); ++q)
      mbar_wait_bounded(&full[q % kStages], static_cast<unsigned>((q / kStages) & 1));
  }
}

__global__ void __launch_bounds__(kRegThreads, 2)
    combine_reg_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                       const int32_t *__restrict__ slot_pos, const float *__restrict__ w,
                       uint4 *__restrict__ out, long n_rows) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int nchunks = (Hv + 31) / 32;
  const long items = static_cast<long>(T) * nchunks;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long it = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int t = static_cast<int>(it / nchunks);
    const int c = static_cast<int>(it - static_cast<long>(t) * nchunks);
    const long tk = static_cast<long>(t) * k;
    const int sp = lane < k ? __ldg(slot_pos + tk + lane) : -1;
    const float wt = lane < k ? (w != nullptr ? __ldg(w + tk + lane) : 1.0f) : 0.0f;
    const int v = c * 32 + lane;

    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
    for (int j0 = 0; j0 < k; j0 += kSlotBatch) {
      uint4 val[kSlotBatch];
      float wj[kSlotBatch];
      bool ok[kSlotBatch];
#pragma unroll
      for (int jj = 0; jj < kSlotBatch; ++jj) {
        const int j = j0 + jj;
        const int row = __shfl_sync(0xffffffffu, sp, j & 31);
        wj[jj] = __shfl_sync(0xffffffffu, wt, j & 31);
        ok[jj] = j < k && row >= 0 && row < n_rows;
        val[jj] = ok[jj] && v < Hv ? ld_stream_v4(y + static_cast<long>(row) * Hv + v)
                                   : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int jj = 0; jj < kSlotBatch; ++jj)
        if (ok[jj]) fma_bf16x8(acc, wj[jj], val[jj]);  // dropped slots add nothing
    }
    if (v < Hv) st_stream_v4(out + static_cast<long>(t) * Hv + v, to_bf16x8(acc));
  }
}

}  // namespace

cudaError_t launch_combine(const void *y, int T, int H, int k, const int32_t *slot_pos,
                           const float *w, void *out, int num_sms, int32_t *d_err,
                           cudaStream_t s, int *launches) {
  const int Hv = H / 8;
  const long n_rows = static_cast<long>(T) * k;
  if (k <= kBulkMaxK) {
    const long items = static_cast<long>(T) * ((Hv + kChunkVec - 1) / kChunkVec);
    if (items == 0) return cudaSuccess;
    const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(combine_bulk_kernel),
                                               kBulkSmem);
    if (err != cudaSuccess) return err;
    // CTAs: one per item, capped at the CTAs that fit on the SMs at once
    const long grid = persistent_grid(reinterpret_cast<const void *>(combine_bulk_kernel),
                                      kChunkVec, kBulkSmem, items * (kChunkVec / kWarp),
                                      num_sms);
    ++*launches;
    return launch_pdl(combine_bulk_kernel, dim3(grid), dim3(kChunkVec), kBulkSmem, s, 1,
                      static_cast<const uint4 *>(y), T, Hv, k, slot_pos, w,
                      static_cast<uint4 *>(out), n_rows, d_err);
  }
  const long items = static_cast<long>(T) * ((Hv + 31) / 32);
  if (items == 0) return cudaSuccess;
  const long grid = persistent_grid(reinterpret_cast<const void *>(combine_reg_kernel),
                                    kRegThreads, 0, items, num_sms);
  ++*launches;
  return launch_pdl(combine_reg_kernel, dim3(grid), dim3(kRegThreads), 0, s, 1,
                    static_cast<const uint4 *>(y), T, Hv, k, slot_pos, w,
                    static_cast<uint4 *>(out), n_rows);
}

}  // namespace ep
