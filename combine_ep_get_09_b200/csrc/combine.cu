// combine.cu -- gate-weighted sum of the expert outputs back into token
// order: out[t] = bf16(fma chain over slots j = 0..k-1 of w[t,j] * y[row]),
// every w[t,j] = 1 when no weights are given (a plain sum, as combining
// per-rank partial outputs needs).
//
// All kernels here run the same fp32 fma chain in slot order, so their
// results are bit-identical to one another:
//
//  * combine_item_kernel (k <= 8; every batch on all SMs): one work item
//    (token t, chunk of 64 16-byte vectors) per CTA of 64 threads.  Every
//    thread reads the token's slot rows and weights (broadcast loads),
//    then its vector of the k rows straight into registers, folds them and
//    writes one vector of the output.  The grid holds every item, so waves
//    of CTAs follow one another as SMs free up; measured against the
//    persistent bulk-copy pipeline below, 96.5 -> 88.1 us inside the
//    prefill step (73 -> 70 us alone) and 3.59 -> 2.88 us a decode call.
//  * combine_bulk_kernel<256> (k <= 8 under an SM budget, num_sms > 0, once
//    the items no longer fit kSmallItemCtasPerSm CTAs per budgeted SM): a
//    bulk-copy (TMA) pipeline on a persistent grid sized to the budget.  A
//    CTA of 256 threads walks a contiguous range of (token, 256-vector
//    chunk) items, the ranges of all CTAs equal to within one item.  Lanes
//    0..k-1 of warp 0 read the token's slot rows and weights and each
//    gathers its row's chunk into shared memory with cp.async.bulk
//    (completing on the stage's mbarrier), kStages items ahead; every
//    thread then folds its 16 bytes of the k rows and writes one 16-byte
//    vector of the output.
//  * combine_reg_kernel (any k <= 32): a warp per item with 128-bit loads
//    of 8 slot rows at a time into registers.
//  * combine_fp8_item_kernel / combine_fp8_bulk_kernel /
//    combine_fp8_reg_kernel: the same for expert outputs kept as e4m3
//    codes plus block scales (below); the item kernel on all SMs (k <= 8),
//    the bulk-copy pipeline under an SM budget (k <= 8, H % 512 == 0).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "bulk.cuh"
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kRegThreads = 256;
constexpr int kSlotBatch = 8;    // slot rows loaded together (register path)
constexpr int kBulkMaxK = 8;     // slot rows one bulk stage holds
// Items in flight per CTA.  Deeper rings measured slower at the prefill
// shape (alone: 77.8 us with 2 stages of 4 KB chunks, 82.0 with 3 stages
// of 2 KB, 88.1 with 3 of 4 KB, 141 with one CTA per SM and 6 stages).
constexpr int kStages = 2;
// 16-byte vectors per row chunk (= threads of the bulk kernel): 256; the
// item kernel takes items of 64 vectors (128 and 256 measured 0.5-3 us
// slower at the prefill shape).
constexpr int kChunkVec = 256;
constexpr int kSmallChunkVec = 64;
constexpr int kSmallItemCtasPerSm = 13;
constexpr long kMaxGridX = 2147483647;  // largest gridDim.x
template <int CHV>
constexpr int bulk_smem() { return kStages * kBulkMaxK * CHV * 16; }

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

template <int kChunkVec>
__global__ void __launch_bounds__(kChunkVec)
    combine_bulk_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                        const int32_t *__restrict__ slot_pos, const float *__restrict__ w,
                        uint4 *__restrict__ out, long n_rows, int first_polls,
                        int32_t *d_err) {
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
    // every expert-output row is read once: evict it first, which left L2
    // to the rest and took the prefill combine from 85 to 78 us
    if (r >= 0)
      bulk_load(stage_buf + (s * kBulkMaxK + lane) * kChunkVec, y + static_cast<long>(r) * Hv + v0,
                bytes, &full[s], l2_policy_evict_first());
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
    const bool ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kStages) & 1),
                                      i == 0 ? first_polls : kMaxBarrierPolls);
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

// One CTA of kSmallChunkVec threads per (token, chunk of kSmallChunkVec
// 16-byte vectors): the slot rows and weights are read by every thread
// (broadcast loads), then each thread loads its vector of the k rows
// straight into registers, so the CTA's chain is two round trips with no
// shared memory or barrier.  Launched with one CTA per item.
__global__ void __launch_bounds__(kSmallChunkVec)
    combine_item_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                        const int32_t *__restrict__ slot_pos, const float *__restrict__ w,
                        uint4 *__restrict__ out, long n_rows) {
  const int nchunks = (Hv + kSmallChunkVec - 1) / kSmallChunkVec;
  const int t = blockIdx.x / nchunks;
  const int v = (blockIdx.x - t * nchunks) * kSmallChunkVec + threadIdx.x;
  pdl_wait();
  const long tk = static_cast<long>(t) * k;
  int row[kBulkMaxK];
  float wj[kBulkMaxK];
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j) {
    row[j] = j < k ? __ldg(slot_pos + tk + j) : -1;
    wj[j] = j < k ? (w != nullptr ? __ldg(w + tk + j) : 1.0f) : 0.0f;
  }
  if (v >= Hv) return;
  uint4 val[kBulkMaxK];
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j)
    val[j] = row[j] >= 0 && row[j] < n_rows ? ld_stream_v4(y + static_cast<long>(row[j]) * Hv + v)
                                            : make_uint4(0, 0, 0, 0);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j)
    if (row[j] >= 0 && row[j] < n_rows) fma_bf16x8(acc, wj[j], val[j]);  // dropped: nothing
  st_stream_v4(out + static_cast<long>(t) * Hv + v, to_bf16x8(acc));
}

__global__ void __launch_bounds__(kRegThreads, 2)
    combine_reg_kernel(const uint4 *__restrict__ y, int T, int Hv, int k,
                       const int32_t *__restrict__ slot_pos, const float *__restrict__ w,
                       uint4 *__restrict__ out, long n_rows) {
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

// ------------------------------------------------------------ FP8 combine
//
// Expert outputs in the FP8 form of dispatch: e4m3 codes y_q [rows, H] and
// one fp32 scale per row and 128-channel block.  Each value is decoded
// (exact), multiplied by its scale in fp32 (round to nearest) and folded
// into the same fp32 fma chain in slot order as the bf16 combine.

// 16 e4m3 codes -> 16 floats (exact: every e4m3 value is a half).
__device__ __forceinline__ void decode_e4m3x16(uint4 v, float *f) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair =
          static_cast<__nv_fp8x2_storage_t>((in[i] >> (16 * h)) & 0xffffu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      const float2 ff = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
      f[4 * i + 2 * h] = ff.x;
      f[4 * i + 2 * h + 1] = ff.y;
    }
  }
}

// Packed pairs of fp32 values (sm_100 f32x2 instructions): each lane of
// fma.rn.f32x2 / mul.rn.f32x2 rounds exactly as the scalar fma.rn.f32 /
// mul.rn.f32 does, so the chains below are the scalar ones, two at a time
// (the FP8 combine is issue-bound: 52.6 -> 48.4 us alone at the prefill
// shape, outputs identical).
__device__ __forceinline__ unsigned long long f2_pack(float a, float b) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ void f2_unpack(unsigned long long d, float *a, float *b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(*a), "=f"(*b) : "l"(d));
}
__device__ __forceinline__ unsigned long long f2_fma(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ void fma_e4m3x16(float *acc, float w, uint4 q, float scale) {
  float f[16];
  decode_e4m3x16(q, f);
  const unsigned long long w2 = f2_pack(w, w), s2 = f2_pack(scale, scale);
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const unsigned long long a = f2_fma(w2, f2_mul(f2_pack(f[e], f[e + 1]), s2),
                                        f2_pack(acc[e], acc[e + 1]));
    f2_unpack(a, &acc[e], &acc[e + 1]);
  }
}

__device__ __forceinline__ void store_bf16x16(uint4 *dst, const float *acc) {
  st_stream_v4(dst, to_bf16x8(acc));
  st_stream_v4(dst + 1, to_bf16x8(acc + 8));
}

constexpr int kQChunkVec = 256;  // 16-byte code vectors (4096 channels) per item
constexpr int kQStageBytes = kBulkMaxK * (kQChunkVec * 16 + kQChunkVec / 8 * 4);
constexpr int kQBulkSmem = kStages * kQStageBytes;

// Bulk-copy pipeline as combine_bulk_kernel (k <= 8; H % 512 == 0 so every
// chunk's codes and scales are whole 16-byte units): item = (token, chunk
// of 4096 channels); lane j < k of warp 0 gathers slot row j's codes and
// its 32 block scales; thread v folds 16 channels of every row.
__global__ void __launch_bounds__(kQChunkVec)
    combine_fp8_bulk_kernel(const uint4 *__restrict__ y_q, const float *__restrict__ y_scale,
                            int T, int H, int k, const int32_t *__restrict__ slot_pos,
                            const float *__restrict__ w, uint4 *__restrict__ out, long n_rows,
                            int first_polls, int32_t *d_err) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ __align__(8) uint64_t full[kStages];
  __shared__ int stage_row[kStages][kBulkMaxK];
  __shared__ float stage_w[kStages][kBulkMaxK];

  const int tid = threadIdx.x, lane = tid & 31;
  const int Hq = H >> 4;  // code vectors per row
  const int nb = H >> 7;  // scales per row
  const int nchunks = (Hq + kQChunkVec - 1) / kQChunkVec;
  const long items = static_cast<long>(T) * nchunks;
  const long first = items * blockIdx.x / gridDim.x;
  const long n_mine = items * (blockIdx.x + 1) / gridDim.x - first;
  auto codes = [&](int s, int j) {
    return reinterpret_cast<uint4 *>(smem_raw + s * kQStageBytes) + j * kQChunkVec;
  };
  auto scales = [&](int s, int j) {
    return reinterpret_cast<float *>(smem_raw + s * kQStageBytes +
                                     kBulkMaxK * kQChunkVec * 16) +
           j * (kQChunkVec / 8);
  };

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&full[s], kWarp);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();

  auto issue = [&](long i) {  // warp 0, as in combine_bulk_kernel
    const long it = first + i;
    const int s = static_cast<int>(i % kStages);
    const int t = static_cast<int>(it / nchunks);
    const int v0 = static_cast<int>(it % nchunks) * kQChunkVec;
    const int nv = min(kQChunkVec, Hq - v0);
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
    const unsigned code_bytes = static_cast<unsigned>(nv) * 16u;
    const unsigned scale_bytes = static_cast<unsigned>(nv / 8) * 4u;
    mbar_arrive_expect_tx(&full[s], r >= 0 ? code_bytes + scale_bytes : 0u);
    if (r >= 0) {  // rows read once: evict first, as in combine_bulk_kernel
      const uint64_t pol = l2_policy_evict_first();
      bulk_load(codes(s, lane), y_q + static_cast<long>(r) * Hq + v0, code_bytes, &full[s], pol);
      bulk_load(scales(s, lane), y_scale + static_cast<long>(r) * nb + v0 / 8, scale_bytes,
                &full[s], pol);
    }
  };

  if (tid < kWarp)
    for (long i = 0; i < min(static_cast<long>(kStages), n_mine); ++i) issue(i);

  long i = 0;
  bool timed_out = false;
  for (; i < n_mine; ++i) {
    const int s = static_cast<int>(i % kStages);
    const long it = first + i;
    const int t = static_cast<int>(it / nchunks);
    const int v0 = static_cast<int>(it % nchunks) * kQChunkVec;
    const bool ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kStages) & 1),
                                      i == 0 ? first_polls : kMaxBarrierPolls);
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    if (tid < Hq - v0) {
      float acc[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int j = 0; j < kBulkMaxK; ++j)
        if (stage_row[s][j] >= 0)
          fma_e4m3x16(acc, stage_w[s][j], codes(s, j)[tid], scales(s, j)[tid >> 3]);
      store_bf16x16(out + (static_cast<long>(t) * Hq + v0 + tid) * 2, acc);
    }
    __syncthreads();  // stage s fully read
    if (tid < kWarp && i + kStages < n_mine) issue(i + kStages);
  }
  if (timed_out && tid == 0) {
    if (d_err != nullptr) atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_TIMEOUT);
    for (long q = i; q < min(n_mine, i + kStages); ++q)
      mbar_wait_bounded(&full[q % kStages], static_cast<unsigned>((q / kStages) & 1));
  }
}

// k <= 8 and H % 128 == 0, one CTA of kSmallChunkVec threads per (token,
// chunk of kSmallChunkVec code vectors = 1024 channels), as
// combine_item_kernel: every thread reads the token's slot rows and
// weights, then its 16 codes and their block scale of each of the k rows
// straight into registers, and writes 16 channels of the output.
__global__ void __launch_bounds__(kSmallChunkVec)
    combine_fp8_item_kernel(const uint4 *__restrict__ y_q, const float *__restrict__ y_scale,
                            int T, int H, int k, const int32_t *__restrict__ slot_pos,
                            const float *__restrict__ w, uint4 *__restrict__ out,
                            long n_rows) {
  const int Hq = H >> 4, nb = H >> 7;
  const int nchunks = (Hq + kSmallChunkVec - 1) / kSmallChunkVec;
  const int t = blockIdx.x / nchunks;
  const int v = (blockIdx.x - t * nchunks) * kSmallChunkVec + threadIdx.x;
  pdl_wait();
  const long tk = static_cast<long>(t) * k;
  int row[kBulkMaxK];
  float wj[kBulkMaxK];
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j) {
    const int r = j < k ? __ldg(slot_pos + tk + j) : -1;
    row[j] = r >= 0 && r < n_rows ? r : -1;  // dropped or out of range: nothing
    wj[j] = j < k ? (w != nullptr ? __ldg(w + tk + j) : 1.0f) : 0.0f;
  }
  if (v >= Hq) return;
  uint4 q[kBulkMaxK];
  float sc[kBulkMaxK];
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j) {
    q[j] = row[j] >= 0 ? ld_stream_v4(y_q + static_cast<long>(row[j]) * Hq + v)
                       : make_uint4(0, 0, 0, 0);
    sc[j] = row[j] >= 0 ? __ldg(y_scale + static_cast<long>(row[j]) * nb + (v >> 3)) : 0.0f;
  }
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
#pragma unroll
  for (int j = 0; j < kBulkMaxK; ++j)
    if (row[j] >= 0) fma_e4m3x16(acc, wj[j], q[j], sc[j]);
  store_bf16x16(out + (static_cast<long>(t) * Hq + v) * 2, acc);
}

// Any k <= 32 and H % 128 == 0: a warp per (token, 512 channels), the
// lane's 16 codes and their scale read directly.
__global__ void __launch_bounds__(kRegThreads, 2)
    combine_fp8_reg_kernel(const uint4 *__restrict__ y_q, const float *__restrict__ y_scale,
                           int T, int H, int k, const int32_t *__restrict__ slot_pos,
                           const float *__restrict__ w, uint4 *__restrict__ out,
                           long n_rows) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int Hq = H >> 4, nb = H >> 7;
  const int nchunks = (Hq + 31) / 32;
  const long items = static_cast<long>(T) * nchunks;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long it = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int t = static_cast<int>(it / nchunks);
    const int v = static_cast<int>(it - static_cast<long>(t) * nchunks) * 32 + lane;
    const long tk = static_cast<long>(t) * k;
    const int sp = lane < k ? __ldg(slot_pos + tk + lane) : -1;
    const float wt = lane < k ? (w != nullptr ? __ldg(w + tk + lane) : 1.0f) : 0.0f;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xffffffffu, sp, j);
      const float wj = __shfl_sync(0xffffffffu, wt, j);
      if (row < 0 || row >= n_rows || v >= Hq) continue;
      fma_e4m3x16(acc, wj, ld_stream_v4(y_q + static_cast<long>(row) * Hq + v),
                  __ldg(y_scale + static_cast<long>(row) * nb + (v >> 3)));
    }
    if (v < Hq) store_bf16x16(out + (static_cast<long>(t) * Hq + v) * 2, acc);
  }
}

}  // namespace

cudaError_t launch_combine_fp8(const void *y_q, const float *y_scale, long n_rows, int T,
                               int H, int k, const int32_t *slot_pos, const float *w,
                               void *out, int num_sms, int32_t *d_err, cudaStream_t s,
                               int *launches) {
  const int Hq = H / 16;
  if (k <= kBulkMaxK && num_sms <= 0) {
    // all SMs: one CTA per item (waves of CTAs follow one another)
    const long items = static_cast<long>(T) * ((Hq + kSmallChunkVec - 1) / kSmallChunkVec);
    if (items == 0) return cudaSuccess;
    if (items <= kMaxGridX) {
      ++*launches;
      return launch_pdl(combine_fp8_item_kernel, dim3(items), dim3(kSmallChunkVec), 0, s, 1,
                        static_cast<const uint4 *>(y_q), y_scale, T, H, k, slot_pos, w,
                        static_cast<uint4 *>(out), n_rows);
    }
  }
  if (k <= kBulkMaxK && H % 512 == 0 && reinterpret_cast<uintptr_t>(y_scale) % 16 == 0) {
    const long items = static_cast<long>(T) * ((Hq + kQChunkVec - 1) / kQChunkVec);
    if (items == 0) return cudaSuccess;
    const cudaError_t err = raise_dynamic_smem(
        reinterpret_cast<const void *>(combine_fp8_bulk_kernel), kQBulkSmem);
    if (err != cudaSuccess) return err;
    const long grid = persistent_grid(reinterpret_cast<const void *>(combine_fp8_bulk_kernel),
                                      kQChunkVec, kQBulkSmem, items * (kQChunkVec / kWarp),
                                      num_sms);
    ++*launches;
    return launch_pdl(combine_fp8_bulk_kernel, dim3(grid), dim3(kQChunkVec), kQBulkSmem, s, 1,
                      static_cast<const uint4 *>(y_q), y_scale, T, H, k, slot_pos, w,
                      static_cast<uint4 *>(out), n_rows, first_wait_polls(), d_err);
  }
  const long items = static_cast<long>(T) * ((Hq + 31) / 32);
  if (items == 0) return cudaSuccess;
  const long grid = persistent_grid(reinterpret_cast<const void *>(combine_fp8_reg_kernel),
                                    kRegThreads, 0, items, num_sms);
  ++*launches;
  return launch_pdl(combine_fp8_reg_kernel, dim3(grid), dim3(kRegThreads), 0, s, 1,
                    static_cast<const uint4 *>(y_q), y_scale, T, H, k, slot_pos, w,
                    static_cast<uint4 *>(out), n_rows);
}

cudaError_t launch_combine(const void *y, long n_rows, int T, int H, int k,
                           const int32_t *slot_pos, const float *w, void *out, int num_sms,
                           int32_t *d_err, cudaStream_t s, int *launches) {
  const int Hv = H / 8;
  if (k <= kBulkMaxK) {
    auto launch = [&](auto kern, int chv, long items, long grid) -> cudaError_t {
      ++*launches;
      return launch_pdl(kern, dim3(grid), dim3(chv), chv * kStages * kBulkMaxK * 16, s, 1,
                        static_cast<const uint4 *>(y), T, Hv, k, slot_pos, w,
                        static_cast<uint4 *>(out), n_rows, first_wait_polls(), d_err);
    };
    if (T == 0) return cudaSuccess;
    {  // one CTA per item of 64 vectors, loaded straight into registers: on
       // all SMs at any size; under an SM budget only while the items fit
       // kSmallItemCtasPerSm CTAs per budgeted SM (a grid of more CTAs
       // would spread over every SM)
      const long items = static_cast<long>(T) * ((Hv + kSmallChunkVec - 1) / kSmallChunkVec);
      const bool fits = num_sms > 0
                            ? items <= static_cast<long>(num_sms) * kSmallItemCtasPerSm
                            : items <= kMaxGridX;
      if (fits) {
        ++*launches;
        return launch_pdl(combine_item_kernel, dim3(items), dim3(kSmallChunkVec), 0, s, 1,
                          static_cast<const uint4 *>(y), T, Hv, k, slot_pos, w,
                          static_cast<uint4 *>(out), n_rows);
      }
    }
    auto kern = combine_bulk_kernel<kChunkVec>;
    constexpr int smem = bulk_smem<kChunkVec>();
    const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern), smem);
    if (err != cudaSuccess) return err;
    const long items = static_cast<long>(T) * ((Hv + kChunkVec - 1) / kChunkVec);
    // CTAs: one per item, capped at the CTAs that fit on the SMs at once
    const long grid = persistent_grid(reinterpret_cast<const void *>(kern), kChunkVec, smem,
                                      items * (kChunkVec / kWarp), num_sms);
    return launch(kern, kChunkVec, items, grid);
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
