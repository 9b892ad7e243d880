// fp8.cuh -- the per-token, per-128-channel FP8 (e4m3) cast of a bf16 row,
// shared by the dispatch kernels: amax of the block, scale = amax / 448
// (fp32, round to nearest), codes = e4m3(x / scale) with the IEEE fp32
// quotient and the hardware round-to-nearest-even, saturating conversion.
// DeepEP's feature list (chinainews.com item; Wallstreetcn review of the
// release) names FP8 dispatch without giving its arithmetic; the amax floor
// of 1e-4 keeps an all-zero block's scale finite.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace ep {

// Largest |value| of 8 bf16 values as a bf16 bit pattern: with the sign
// cleared, bf16 bit patterns order like their magnitudes (NaN above inf), so
// an unsigned max of the patterns is the max of |x| with NaN propagating.
__device__ __forceinline__ uint32_t absmax_bits_bf16x8(uint4 v) {
  const uint32_t a = __vmaxu2(v.x & 0x7fff7fffu, v.y & 0x7fff7fffu);
  const uint32_t b = __vmaxu2(v.z & 0x7fff7fffu, v.w & 0x7fff7fffu);
  const uint32_t m = __vmaxu2(a, b);
  return max(m & 0xffffu, m >> 16);
}

// e4m3 codes of x / s for 8 bf16 values: IEEE fp32 quotient (round to
// nearest), then the hardware e4m3 conversion (round to nearest even,
// saturating to +-448).
__device__ __forceinline__ uint2 quantize_bf16x8(uint4 v, float s) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(in[i] << 16);
    const float hi = __uint_as_float(in[i] & 0xffff0000u);
    q[i] = __nv_cvt_float2_to_fp8x2(make_float2(__fdiv_rn(lo, s), __fdiv_rn(hi, s)),
                                    __NV_SATFINITE, __NV_E4M3);
  }
  return make_uint2(q[0] | (q[1] << 16), q[2] | (q[3] << 16));
}

// amax -> scale -> e4m3 for the 8 bf16 values of one lane, the lane being
// one of the 16 lanes (a half-warp) that hold a 128-channel block.
__device__ __forceinline__ uint2 quantize_block_lane(uint4 v, float *scale) {
  uint32_t m = absmax_bits_bf16x8(v);
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  float a = __uint_as_float(m << 16);
  a = a < 1e-4f ? 1e-4f : a;  // keeps NaN
  *scale = __fdiv_rn(a, 448.0f);
  return quantize_bf16x8(v, *scale);
}

}  // namespace ep
