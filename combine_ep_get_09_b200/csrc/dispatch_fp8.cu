// dispatch_fp8.cu -- token rows to expert-contiguous receive rows with the
// FP8 cast (e4m3 codes, one fp32 scale per token and 128-channel block)
// fused in: a bulk-copy kernel for hidden sizes that are multiples of 512
// and a register kernel for the other multiples of 128.  Both read each
// source byte once and write each destination byte once.
#include <algorithm>

#include "bulk.cuh"
#include "ep_internal.cuh"
#include "fp8.cuh"

namespace ep {
namespace {

constexpr int kThreads = 256;  // register kernel

constexpr int kFp8BulkThreads = 256;
// bf16 rows in flight per CTA: two on a persistent grid (a CTA walking a
// token range loads the next row while it casts this one), one when every
// token has a CTA of its own (8 CTAs per SM instead of 6: 54.2-55.3 ->
// 53.3-54.2 us inside the prefill step)
constexpr int kFp8InStagesRange = 2;
constexpr int kFp8InStagesOne = 1;
// Cast rows whose bulk stores may still be reading them.  Two measured
// slower at the prefill shape (59.5 vs 57.5 us alone): the extra stage
// costs a CTA per SM (5 instead of 6), which hurts more than the overlap
// helps; so did one input stage with two or three output stages (63.5 and
// 59.4 us).
constexpr int kFp8OutStages = 1;

// FP8 dispatch through shared memory, one token row per item (H a
// multiple of 512, so that both the e4m3 row and its H/128 scales are
// whole 16-byte units): thread 0 bulk-loads the rows kFp8InStages ahead,
// the CTA quantizes the current one into an output stage (half-warp per
// 128-channel block), and thread 0 bulk-stores that stage to each of the
// token's k receive rows (codes and scales).  Whole-row bulk stores write
// HBM better than per-lane stores (measured at the prefill shape: 55 us
// against 57 us for 16-byte stores per lane, 59 us for 512-byte bulk
// stores per warp, and 61 us for half-row items).
// At H = 7168, 6 CTAs of 256 threads with two input stages fit an SM's
// shared memory, 8 with one; the bound keeps registers low enough that
// they fit too.
template <int kFp8InStages>
__global__ void __launch_bounds__(kFp8BulkThreads, kFp8InStages == 1 ? 8 : 6)
    dispatch_fp8_bulk_kernel(const uint4 *__restrict__ x, int T, int H, int k,
                             const int32_t *__restrict__ slot_pos, uint8_t *__restrict__ recv_q,
                             float *__restrict__ recv_scale, long n_rows, int first_polls,
                             int32_t *d_err) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int in_bytes = 2 * H, q_bytes = H, nb = H >> 7, s_bytes = 4 * nb;
  const int out_bytes = q_bytes + s_bytes;                           // a multiple of 16
  unsigned char *in_buf = smem_raw;                                  // [in stages][2H]
  unsigned char *out_buf = smem_raw + kFp8InStages * in_bytes;       // [out stages][H + H/32]
  __shared__ __align__(8) uint64_t full[kFp8InStages];
  __shared__ int rows[2][EP_MAX_K];
  const int tid = threadIdx.x;
  const long items = T;
  // CTA b takes items [b * per, b * per + per): the CTAs that finish early
  // leave their SM to the rest (an even split to within one item keeps
  // every SM's CTAs busy for the same 5-token chains and measured 3 %
  // slower at the prefill shape)
  const long per = (items + gridDim.x - 1) / gridDim.x;
  const long first = min(items, static_cast<long>(blockIdx.x) * per);
  const long n_mine = min(items, first + per) - first;

  // the receive rows are written once and read by a later kernel: evict
  // them first (measured: the step 0.3-0.5 % faster, the kernel ~1 %)
  const uint64_t pol = l2_policy_evict_first();
  if (tid == 0) {
    for (int s = 0; s < kFp8InStages; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
  }
  __syncthreads();
  pdl_wait();

  auto issue = [&](long i) {  // thread 0: token first + i -> input stage i % stages
    const int s = static_cast<int>(i % kFp8InStages);
    mbar_arrive_expect_tx(&full[s], in_bytes);
    bulk_load(in_buf + s * in_bytes, x + (first + i) * (H >> 3), in_bytes, &full[s]);
  };
  if (tid == 0)
    for (long i = 0; i < min(static_cast<long>(kFp8InStages), n_mine); ++i) issue(i);

  long i = 0;
  bool timed_out = false;
  for (; i < n_mine; ++i) {
    const long t = first + i;
    const int s = static_cast<int>(i % kFp8InStages);
    unsigned char *out_q = out_buf + (i % kFp8OutStages) * out_bytes;
    float *out_s = reinterpret_cast<float *>(out_q + q_bytes);
    // the stores of the item that last used this output stage have read it
    if (tid == 0) bulk_wait_read<kFp8OutStages - 1>();
    if (tid < k) rows[i & 1][tid] = __ldg(slot_pos + t * k + tid);
    const bool ok = mbar_wait_bounded(&full[s], static_cast<unsigned>((i / kFp8InStages) & 1),
                                      i == 0 ? first_polls : kMaxBarrierPolls);
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    const uint4 *xin = reinterpret_cast<const uint4 *>(in_buf + s * in_bytes);
    uint2 *qo = reinterpret_cast<uint2 *>(out_q);
    // 16 consecutive vectors = one block per half-warp; whole warps share
    // the loop bound because H / 8 is a multiple of 64
    for (int v = tid; v < (H >> 3); v += kFp8BulkThreads) {
      float sc;
      qo[v] = quantize_block_lane(xin[v], &sc);
      if ((tid & 15) == 0) out_s[v >> 4] = sc;
    }
    fence_proxy_async_smem();  // the stage's generic writes before the bulk reads
    __syncthreads();           // input stage s read, output stage written
    if (tid == 0) {
      if (i + kFp8InStages < n_mine) issue(i + kFp8InStages);
      for (int j = 0; j < k; ++j) {
        const int row = rows[i & 1][j];
        if (row < 0 || row >= n_rows) continue;
        bulk_store(recv_q + static_cast<long>(row) * H, out_q, q_bytes, pol);
        bulk_store(recv_scale + static_cast<long>(row) * nb, out_s, s_bytes, pol);
      }
      bulk_commit();
    }
  }
  if (tid == 0) {
    if (timed_out) {
      if (d_err != nullptr) atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_TIMEOUT);
      // the loads still in flight (items i .. i + stages - 1, the one the
      // wait gave up on included) land before the CTA's memory goes away
      for (long q = i; q < min(n_mine, i + kFp8InStages); ++q)
        mbar_wait_bounded(&full[q % kFp8InStages],
                          static_cast<unsigned>((q / kFp8InStages) & 1));
    }
    // the stores must have read the output stage before the CTA's shared
    // memory goes away; their writes are visible to later kernels once the
    // grid completes
    bulk_wait_read<0>();
  }
}

// Work item = (token, chunk of 4 blocks of 128 channels).  Lane l covers
// 8 channels of block 2p + (l >> 4) for p = 0, 1: each half-warp owns a
// block per load, so the amax reduction is 4 xor-shuffles inside it and
// every load / store instruction of the warp touches one contiguous span.
__global__ void __launch_bounds__(kThreads)
    dispatch_fp8_kernel(const uint4 *__restrict__ x, int T, int H, int k,
                        const int32_t *__restrict__ slot_pos,
                        uint2 *__restrict__ recv_q,
                        float *__restrict__ recv_scale, long n_rows) {
  pdl_wait();
  const int lane = threadIdx.x & 31, half = lane >> 4, sub = lane & 15;
  const int Hv = H >> 3;   // 8-channel units per row (16 B in, 8 B out)
  const int nb = H >> 7;   // 128-channel blocks per row
  const int nchunks = (nb + 3) >> 2;
  const long items = static_cast<long>(T) * nchunks;
  const long nwarps = (static_cast<long>(gridDim.x) * blockDim.x) >> 5;
  for (long it = (static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int t = static_cast<int>(it / nchunks);
    const int c = static_cast<int>(it - static_cast<long>(t) * nchunks);
    const int sp = lane < k ? __ldg(slot_pos + static_cast<long>(t) * k + lane) : -1;
    const uint4 *src = x + static_cast<long>(t) * Hv;

    int blk[2];
    bool ok[2];
    uint4 v[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      blk[p] = 4 * c + 2 * p + half;
      ok[p] = blk[p] < nb;
      v[p] = ok[p] ? ld_stream_v4(src + blk[p] * 16 + sub) : make_uint4(0, 0, 0, 0);
    }
    float s[2];
    uint2 q[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      uint32_t m = absmax_bits_bf16x8(v[p]);
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
      float a = __uint_as_float(m << 16);
      a = a < 1e-4f ? 1e-4f : a;  // keeps NaN
      s[p] = __fdiv_rn(a, 448.0f);
      q[p] = quantize_bf16x8(v[p], s[p]);
    }
    for (int j = 0; j < k; ++j) {
      const int row = __shfl_sync(0xffffffffu, sp, j);
      if (row < 0 || row >= n_rows) continue;
      uint2 *dst = recv_q + static_cast<long>(row) * Hv;
#pragma unroll
      for (int p = 0; p < 2; ++p)
        if (ok[p]) st_stream_v2(dst + blk[p] * 16 + sub, q[p]);
    }
    // scales: lane l stores block (l & 3) of the chunk for slot j0 + (l >> 2);
    // block 2p + h's scale sits in s[p] of half h
    const int bb = lane & 3;
    const float s0 = __shfl_sync(0xffffffffu, s[0], (bb & 1) * 16);
    const float s1 = __shfl_sync(0xffffffffu, s[1], (bb & 1) * 16);
    const float sv = (bb >> 1) ? s1 : s0;
    const int b = 4 * c + bb;
    for (int j0 = 0; j0 < k; j0 += 8) {
      const int j = j0 + (lane >> 2);
      const int row = __shfl_sync(0xffffffffu, sp, j & 31);
      if (j < k && b < nb && row >= 0 && row < n_rows)
        st_stream_f32(recv_scale + static_cast<long>(row) * nb + b, sv);
    }
  }
}

}  // namespace

// Largest hidden size the bulk FP8 kernel stages in shared memory.
constexpr int kFp8BulkMaxH = 16384;

int fp8_bulk_smem(int in_stages, int H) {
  return in_stages * 2 * H + kFp8OutStages * (H + H / 32);
}

cudaError_t launch_dispatch_fp8(const void *x, int T, int H, int k,
                                const int32_t *slot_pos, void *recv_q,
                                float *recv_scale, long n_rows, int num_sms, int32_t *d_err,
                                cudaStream_t s, int *launches) {
  // bulk stores need 16-byte aligned scale rows: H % 512 == 0 and an
  // aligned recv_scale
  if (H % 512 == 0 && H <= kFp8BulkMaxH && reinterpret_cast<uintptr_t>(recv_scale) % 16 == 0) {
    if (T == 0) return cudaSuccess;
    // all SMs: one token per CTA, waves of CTAs following one another as
    // SMs free up (measured against a persistent grid of 6 CTAs per SM:
    // 57.5-62 -> 54.2-55.3 us inside the prefill step, 49-52 -> 46-47 us
    // alone); under an SM budget a persistent grid sized to it
    auto launch = [&](auto kern, int in_stages, long grid) -> cudaError_t {
      const cudaError_t err = raise_dynamic_smem(reinterpret_cast<const void *>(kern),
                                                 fp8_bulk_smem(in_stages, kFp8BulkMaxH));
      if (err != cudaSuccess) return err;
      ++*launches;
      return launch_pdl(kern, dim3(grid), dim3(kFp8BulkThreads), fp8_bulk_smem(in_stages, H), s,
                        1, static_cast<const uint4 *>(x), T, H, k, slot_pos,
                        static_cast<uint8_t *>(recv_q), recv_scale, n_rows, first_wait_polls(),
                        d_err);
    };
    if (num_sms <= 0)
      return launch(dispatch_fp8_bulk_kernel<kFp8InStagesOne>, kFp8InStagesOne,
                    static_cast<long>(T));
    auto kern = dispatch_fp8_bulk_kernel<kFp8InStagesRange>;
    const long grid = persistent_grid(reinterpret_cast<const void *>(kern), kFp8BulkThreads,
                                      fp8_bulk_smem(kFp8InStagesRange, H),
                                      static_cast<long>(T) * (kFp8BulkThreads / kWarp), num_sms);
    return launch(kern, kFp8InStagesRange, grid);
  }
  const long nchunks = (H / 128 + 3) / 4;
  const long items = static_cast<long>(T) * nchunks;
  if (items == 0) return cudaSuccess;
  // a warp per item: one CTA per kThreads / 32 items on all SMs, a
  // persistent grid under an SM budget
  constexpr long kWarpsPerCta = kThreads / 32;
  const long grid = num_sms > 0
                        ? persistent_grid(reinterpret_cast<const void *>(dispatch_fp8_kernel),
                                          kThreads, 0, items, num_sms)
                        : std::min((items + kWarpsPerCta - 1) / kWarpsPerCta, 2147483647L);
  ++*launches;
  return launch_pdl(dispatch_fp8_kernel, dim3(grid), dim3(kThreads), 0, s, 1,
                    static_cast<const uint4 *>(x), T, H, k, slot_pos,
                    static_cast<uint2 *>(recv_q), recv_scale, n_rows);
}

}  // namespace ep
