// layout_noalloc.cu -- ep_get_layout_noalloc: the dispatch layout for
// callers that cannot allocate device memory (a runtime whose memory is
// all owned by its own pool, or a loop that must not pay cudaMalloc's
// implicit synchronisation).  The tiled layout's scratch (a 16-byte ticket
// plus one row of E + R counters per tile of tokens) lives in a fixed
// array defined here instead of a caller workspace; the kernels are the
// ones ep_get_layout launches.
#include "ep_internal.cuh"

namespace {

// One copy per device (per context), from module load until the process
// exits; zero-filled when the module is loaded.
static __device__ __align__(256) unsigned char g_layout_scratch[EP_NOALLOC_SCRATCH_BYTES];

// Device address of g_layout_scratch in the current context.  In host code
// the array's name only stands for the symbol, so the address has to come
// from the runtime.  It is looked up on every call: once the module is
// loaded that is a table lookup, not a stream operation, and it stays
// right for whichever context is current (a non-primary one, or the
// primary one again after cudaDeviceReset).  The first lookup on a device
// loads the module, which is why the first call should precede any stream
// capture.
ep_status_t scratch_address(void **addr) {
  void *p = nullptr;
  const cudaError_t err = cudaGetSymbolAddress(&p, g_layout_scratch);
  if (err != cudaSuccess || p == nullptr)
    return ep::record_error(EP_ERR_CUDA, "ep_get_layout_noalloc: cudaGetSymbolAddress: %s",
                            cudaGetErrorString(err));
  *addr = p;
  return EP_OK;
}

// The scratch array used is the current device's, so the work must run
// there: `stream` must belong to the current device and `idx` must live on
// it (or be reachable as host-mapped or managed memory).
ep_status_t check_device(const void *idx, cudaStream_t stream) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess)
    return ep::record_error(EP_ERR_CUDA, "ep_get_layout_noalloc: cudaGetDevice: %s",
                            cudaGetErrorString(err));
  if (stream != nullptr) {
    int sdev = -1;
    err = cudaStreamGetDevice(stream, &sdev);
    if (err != cudaSuccess)
      return ep::record_error(EP_ERR_INVALID_ARG,
                              "ep_get_layout_noalloc: stream is not a valid stream: %s",
                              cudaGetErrorString(err));
    if (sdev != dev)
      return ep::record_error(EP_ERR_INVALID_ARG,
                              "ep_get_layout_noalloc: stream belongs to device %d but the "
                              "current device is %d (the scratch used is the current "
                              "device's); make device %d current first",
                              sdev, dev, sdev);
  }
  cudaPointerAttributes attr = {};
  err = cudaPointerGetAttributes(&attr, idx);
  if (err != cudaSuccess) {
    cudaGetLastError();  // a plain host pointer is not an error to keep
    return ep::record_error(EP_ERR_INVALID_ARG,
                            "ep_get_layout_noalloc: idx is not device memory: %s",
                            cudaGetErrorString(err));
  }
  if (attr.type == cudaMemoryTypeDevice && attr.device != dev)
    return ep::record_error(EP_ERR_INVALID_ARG,
                            "ep_get_layout_noalloc: idx is on device %d but the current "
                            "device is %d; make device %d current first",
                            attr.device, dev, attr.device);
  if (attr.type == cudaMemoryTypeUnregistered || attr.type == cudaMemoryTypeHost) {
    if (attr.devicePointer == nullptr)
      return ep::record_error(EP_ERR_INVALID_ARG,
                              "ep_get_layout_noalloc: idx is host memory the device cannot "
                              "reach");
  }
  return EP_OK;
}

}  // namespace

extern "C" ep_status_t ep_get_layout_noalloc(const void *idx, int idx_is_int64, int T,
                                             int k, int E, int R, int32_t *cnt_e,
                                             int32_t *cnt_r, uint8_t *in_rank,
                                             int32_t *off_e, int32_t *off_r,
                                             int32_t *slot_pos, int32_t *recv_src,
                                             int32_t *d_err, void *stream) {
  // every check comes before anything is enqueued
  ep_status_t st = ep::check_layout_args("ep_get_layout_noalloc", idx, idx_is_int64, T, k,
                                         E, R, cnt_e, cnt_r, in_rank, off_e, off_r,
                                         slot_pos, recv_src, d_err);
  if (st != EP_OK) return st;
  const size_t need = ep_layout_workspace_bytes(T, k, E, R);
  if (need > EP_NOALLOC_SCRATCH_BYTES)
    return ep::record_error(
        EP_ERR_UNSUPPORTED,
        "ep_get_layout_noalloc: T=%d k=%d E=%d R=%d needs %zu bytes of scratch, "
        "more than the library's fixed %u; use ep_get_layout with a workspace",
        T, k, E, R, need, EP_NOALLOC_SCRATCH_BYTES);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T == 0 || need == 0)  // no scratch is touched: plain ep_get_layout
    return ep_get_layout(idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r, in_rank, off_e, off_r,
                         slot_pos, recv_src, nullptr, 0, d_err, stream);
  st = check_device(idx, s);
  if (st != EP_OK) return st;
  void *scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != EP_OK) return st;
  // The array is zero when the module loads, and every call leaves its
  // ticket at zero again (the tiled layout's place kernel clears it after
  // the count kernel), so nothing is cleared here: a clear would be one more
  // node in front of the layout kernels, measured at 3.9 us a call.
  return ep_get_layout(idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r, in_rank, off_e, off_r,
                       slot_pos, recv_src, scratch, EP_NOALLOC_SCRATCH_BYTES, d_err, stream);
}
