// ep_internal.cuh -- launcher declarations and host helpers shared by the
// files of libep.so (internal; the public ABI is include/ep.h; the device
// helpers are in ep_device.cuh).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "ep.h"
#include "ep_device.cuh"

namespace ep {

// --------------------------------------------------------------- launchers
// Each returns cudaSuccess or the launch error; arguments are validated by
// the ABI layer before these are called.

// What LayoutArgs::idx points at.
constexpr int kIdsInt32 = 0;  // int32 expert ids [T, k]
constexpr int kIdsInt64 = 1;  // int64 expert ids [T, k]
constexpr int kIdsMask = 2;   // uint8 mask [T, k]: slot (t, j) is expert j when set

struct LayoutArgs {
  const void *idx;
  int id_kind;
  int T, k, E, R;
  int32_t *cnt_e, *cnt_r, *off_e, *off_r, *slot_pos, *recv_src;
  uint8_t *in_rank;
  void *ws;
  int32_t *d_err;
};

size_t layout_workspace_bytes(int T, int k, int E, int R);
cudaError_t launch_layout(const LayoutArgs &a, cudaStream_t s, int *launches);

// n_rows: rows of the receive buffer; slot rows outside [0, n_rows) are
// skipped.
cudaError_t launch_dispatch_bf16(const void *x, int T, int H, int k,
                                 const int32_t *slot_pos, void *recv, long n_rows,
                                 int num_sms, int32_t *d_err, cudaStream_t s,
                                 int *launches);
cudaError_t launch_dispatch_fp8(const void *x, int T, int H, int k,
                                const int32_t *slot_pos, void *recv_q,
                                float *recv_scale, long n_rows, int num_sms, int32_t *d_err,
                                cudaStream_t s, int *launches);
// Layout and dispatch in one launch (small batches; see layout_dispatch.cu).
// layout_dispatch_fusable says whether the sizes (and, for FP8, the scale
// pointer's alignment) fit that kernel.
bool layout_dispatch_fusable(int T, int k, int E, int R, int H, bool fp8,
                             const float *recv_scale);
cudaError_t launch_layout_dispatch(const LayoutArgs &la, const void *x, int H, bool fp8,
                                   void *recv, float *recv_scale, int num_sms, cudaStream_t s,
                                   int *launches);
cudaError_t launch_combine(const void *y, long n_rows, int T, int H, int k,
                           const int32_t *slot_pos, const float *w, void *out,
                           int num_sms, int32_t *d_err, cudaStream_t s,
                           int *launches);
// FP8 expert outputs: e4m3 codes y_q [n_rows, H] and fp32 scales y_scale
// [n_rows, H / 128].
cudaError_t launch_combine_fp8(const void *y_q, const float *y_scale, long n_rows, int T,
                               int H, int k, const int32_t *slot_pos, const float *w,
                               void *out, int num_sms, int32_t *d_err, cudaStream_t s,
                               int *launches);
// Physical expert of every slot from the logical layout (replicas.cu).
cudaError_t launch_map_replicas(const void *idx, bool int64_ids, int T, int k, int E,
                                const int32_t *slot_pos, const int32_t *off_e,
                                const int32_t *rep_off, const int32_t *rep_ids, int32_t *phys,
                                int32_t *d_err, cudaStream_t s, int *launches);
// Aligned receive segments from a plain layout (pad_layout.cu).
cudaError_t launch_pad_layout(const int32_t *cnt_e, const int32_t *slot_pos, int T, int k,
                              int E, int align, int32_t *off_pad, int32_t *slot_pos_pad,
                              int32_t *recv_src_pad, cudaStream_t s, int *launches);

// Poll limit of the first bounded mbarrier wait of each CTA of the
// bulk-copy kernels: kMaxBarrierPolls, or 0 while the testing switch
// ep_debug_expire_first_wait is on.
int first_wait_polls();

// Sets the message ep_last_error_string() returns on this host thread and
// returns `status` (for entry points defined outside ep_abi.cu).
ep_status_t record_error(ep_status_t status, const char *fmt, ...);

// The argument checks ep_get_layout makes, except those of the workspace.
ep_status_t check_layout_args(const char *fn, const void *idx, int idx_is_int64, int T,
                              int k, int E, int R, const int32_t *cnt_e,
                              const int32_t *cnt_r, const uint8_t *in_rank,
                              const int32_t *off_e, const int32_t *off_r,
                              const int32_t *slot_pos, const int32_t *recv_src,
                              const int32_t *d_err);

// SM count of the current device (cached per device).
int device_sm_count();

// Grid for a persistent kernel: enough blocks of `threads` threads to give
// each of `warp_items` work items a warp, capped at the blocks that fit at
// once (with `smem_bytes` of dynamic shared memory each) on `num_sms` SMs
// (0 = all SMs).  The occupancy figure is cached per (device, kernel,
// threads, shared memory).
long persistent_grid(const void *kernel, int threads, int smem_bytes, long warp_items,
                     int num_sms);

// Largest dynamic shared memory a CTA of `kernel` may opt in to on the
// current device: the device's opt-in limit less the kernel's static shared
// memory (cached per device and kernel).
int max_dynamic_smem(const void *kernel);

// Raises a kernel's dynamic shared memory limit to `bytes` (once per
// device and kernel).
cudaError_t raise_dynamic_smem(const void *kernel, int bytes);

// Launches `kernel` with programmatic stream serialization (see pdl_wait)
// and, when cluster > 1, a thread-block cluster of that many CTAs.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, int smem,
                       cudaStream_t stream, int cluster, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace ep
