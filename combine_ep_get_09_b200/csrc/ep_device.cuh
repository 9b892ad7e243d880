// ep_device.cuh -- device helpers shared by the kernels of libep.so: the
// streaming loads and stores of the row copies, programmatic dependent
// launch, lane masks (internal).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ep {

constexpr int kWarp = 32;

// ---------------------------------------------------------------- memory

// 128-bit read-only load that bypasses L1 allocation: the row is read once
// per launch, so keeping it out of L1 leaves L1 to the index arrays.  The
// DeepEP blog (frogred8, "deepEP optimization", second method) describes
// the same non-coherent, no-allocate read for its communication buffers.
__device__ __forceinline__ uint4 ld_stream_v4(const uint4 *p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// Write-once outputs: streaming stores (evict-first in L1 and L2).
__device__ __forceinline__ void st_stream_v4(uint4 *p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ void st_stream_v2(uint2 *p, uint2 v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x),
               "r"(v.y)
               : "memory");
}

__device__ __forceinline__ void st_stream_f32(float *p, float v) {
  asm volatile("st.global.cs.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// Programmatic dependent launch (sm_90+).  Every kernel of the library is
// launched with programmatic stream serialization, so it may be scheduled
// while the previous kernel on the stream is still finishing; it must call
// pdl_wait() before touching memory that kernel writes (griddepcontrol.wait
// returns once the previous grid has completed and its writes are visible;
// with no such predecessor it returns at once).  Almost no kernel issues
// griddepcontrol.launch_dependents: a CTA's exit counts as its trigger, so
// the next kernel is launched as this one's last CTAs leave, which hides
// its launch latency without parking its CTAs on SMs that are still busy.
// (Triggering at kernel entry measured slower everywhere: 288 vs 256 us
// for a back-to-back prefill step, 8.23 vs 8.12 us for a decode call.)
// The one exception, the one-token-per-CTA fused decode kernel, triggers
// once only its final stores are left (layout_dispatch.cu).
//
// Bulk prefetch of [p, p + bytes) into L2 (p 16-byte aligned, bytes a
// multiple of 16); a hint with no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void *p, int bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

}  // namespace ep
