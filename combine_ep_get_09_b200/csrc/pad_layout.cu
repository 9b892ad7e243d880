// pad_layout.cu -- receive segments aligned for a grouped GEMM.
//
// The dispatch layout packs the experts' receive rows back to back.  A
// grouped GEMM that walks the receive buffer in row tiles of `align` rows
// wants every expert's segment to start on a tile boundary, so that no tile
// mixes two experts; this kernel turns a plain layout into that form:
//   off_pad[e]        = sum over e' < e of ceil(cnt_e[e'] / align) * align
//   slot_pos_pad[t,j] = off_pad[e] + (slot_pos[t,j] - off_e[e])  (same rank)
//   recv_src_pad[r]   = token of padded row r, -1 for padding rows and
//                       past off_pad[E]; T*k + E*(align-1) rows
// Every CTA scans the E counts itself (plain and padded offsets, a few KB of
// shared memory), then walks a grid-stride share of the slots and of the
// padded rows; the expert of a row is found by binary search over the
// offsets.  No CTA waits on another.
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kPadThreads = 256;

// Largest e in [0, E) with off[e] <= v (off ascending, off[0] = 0 <= v).
__device__ __forceinline__ int segment_of(const int *off, int E, int v) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= v)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kPadThreads)
    pad_layout_kernel(const int32_t *__restrict__ cnt_e, const int32_t *slot_pos, int T, int k,
                      int E, int align, int32_t *__restrict__ off_pad, int32_t *slot_pos_pad,
                      int32_t *__restrict__ recv_src_pad, long n_cap) {
  extern __shared__ int smem[];
  int *cnt = smem;          // [E]
  int *off = cnt + E;       // [E + 1] plain offsets
  int *offp = off + E + 1;  // [E + 1] padded offsets
  const int tid = threadIdx.x, lane = tid & 31;

  pdl_wait();
  for (int e = tid; e < E; e += kPadThreads) cnt[e] = __ldg(cnt_e + e);
  __syncthreads();
  if (tid < kWarp) {  // warp 0 scans both offset arrays, 32 experts a round
    int carry = 0, carry_p = 0;
    for (int b = 0; b < E; b += kWarp) {
      const int e = b + lane;
      const int c = e < E ? cnt[e] : 0;
      const int cp = (c + align - 1) / align * align;
      int incl = c, incl_p = cp;
#pragma unroll
      for (int o = 1; o < kWarp; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        const int up = __shfl_up_sync(0xffffffffu, incl_p, o);
        if (lane >= o) {
          incl += u;
          incl_p += up;
        }
      }
      if (e < E) {
        off[e] = carry + incl - c;
        offp[e] = carry_p + incl_p - cp;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
      carry_p += __shfl_sync(0xffffffffu, incl_p, 31);
    }
    if (lane == 0) {
      off[E] = carry;
      offp[E] = carry_p;
    }
  }
  __syncthreads();
  if (blockIdx.x == 0)
    for (int e = tid; e <= E; e += kPadThreads) off_pad[e] = offp[e];

  const long stride = static_cast<long>(gridDim.x) * kPadThreads;
  const long start = static_cast<long>(blockIdx.x) * kPadThreads + tid;
  const long N = static_cast<long>(T) * k;
  const int kept = off[E], kept_p = offp[E];
  // every slot: the same rank inside its expert, at the padded offset
  for (long i = start; i < N; i += stride) {
    const int row = slot_pos[i];
    int out = -1;
    if (row >= 0 && row < kept) {
      const int e = segment_of(off, E, row);
      out = offp[e] + (row - off[e]);
      // slots number fewer than 2^31: an exact 32-bit division
      recv_src_pad[out] = static_cast<int32_t>(static_cast<unsigned>(i) / static_cast<unsigned>(k));
    }
    slot_pos_pad[i] = out;
  }
  // padding rows and rows past the last segment
  for (long r = start; r < n_cap; r += stride) {
    if (r >= kept_p) {
      recv_src_pad[r] = -1;
      continue;
    }
    const int e = segment_of(offp, E, static_cast<int>(r));
    if (r - offp[e] >= cnt[e]) recv_src_pad[r] = -1;
  }
}

}  // namespace

cudaError_t launch_pad_layout(const int32_t *cnt_e, const int32_t *slot_pos, int T, int k,
                              int E, int align, int32_t *off_pad, int32_t *slot_pos_pad,
                              int32_t *recv_src_pad, cudaStream_t s, int *launches) {
  const long n_cap = static_cast<long>(T) * k + static_cast<long>(E) * (align - 1);
  const int smem = (3 * E + 2) * static_cast<int>(sizeof(int));
  const long work = n_cap > static_cast<long>(T) * k ? n_cap : static_cast<long>(T) * k;
  // about 2 elements per thread, at most the CTAs that fit at once
  const long grid = persistent_grid(reinterpret_cast<const void *>(pad_layout_kernel),
                                    kPadThreads, smem, (work + 63) / 64, 0);
  ++*launches;
  return launch_pdl(pad_layout_kernel, dim3(grid > 0 ? grid : 1), dim3(kPadThreads), smem, s, 1,
                    cnt_e, slot_pos, T, k, E, align, off_pad, slot_pos_pad, recv_src_pad, n_cap);
}

}  // namespace ep
