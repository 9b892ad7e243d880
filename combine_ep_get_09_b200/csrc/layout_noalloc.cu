// layout_noalloc.cu -- ep_get_layout_noalloc: the dispatch layout for
// callers that cannot allocate device memory (a runtime whose memory is
// all owned by its own pool, or a loop that must not pay cudaMalloc's
// implicit synchronisation).  The tiled layout's scratch (a 16-byte ticket
// plus one row of E + R counters per tile of tokens) lives in a fixed
// array defined here instead of a caller workspace; the kernels are the
// ones ep_get_layout launches.
#include <mutex>

#include "ep_internal.cuh"

namespace {

// One copy per device, from module load until the process exits.
static __device__ __align__(256) unsigned char g_layout_scratch[EP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kTicketBytes = 16;

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_layout_scratch on the current device.  In host code
// the array's name only stands for the symbol, so the address has to come
// from the runtime; it is looked up once per device and cached.
ep_status_t scratch_address(void **addr) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess)
    return ep::record_error(EP_ERR_CUDA, "ep_get_layout_noalloc: cudaGetDevice: %s",
                            cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices)
    return ep::record_error(EP_ERR_UNSUPPORTED,
                            "ep_get_layout_noalloc: device %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void *p = nullptr;
    err = cudaGetSymbolAddress(&p, g_layout_scratch);
    if (err != cudaSuccess || p == nullptr)
      return ep::record_error(EP_ERR_CUDA,
                              "ep_get_layout_noalloc: cudaGetSymbolAddress: %s",
                              cudaGetErrorString(err));
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return EP_OK;
}

}  // namespace

extern "C" ep_status_t ep_get_layout_noalloc(const void *idx, int idx_is_int64, int T,
                                             int k, int E, int R, int32_t *cnt_e,
                                             int32_t *cnt_r, uint8_t *in_rank,
                                             int32_t *off_e, int32_t *off_r,
                                             int32_t *slot_pos, int32_t *recv_src,
                                             int32_t *d_err, void *stream) {
  // every check comes before any CUDA call
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
  void *scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != EP_OK) return st;
  if (need > 0) {
    // the previous call left its contents; the ticket must start at zero
    const cudaError_t err = cudaMemsetAsync(scratch, 0, kTicketBytes,
                                            static_cast<cudaStream_t>(stream));
    if (err != cudaSuccess)
      return ep::record_error(EP_ERR_CUDA, "ep_get_layout_noalloc: clearing scratch: %s",
                              cudaGetErrorString(err));
  }
  return ep_get_layout(idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r, in_rank, off_e,
                       off_r, slot_pos, recv_src, scratch, EP_NOALLOC_SCRATCH_BYTES,
                       d_err, stream);
}
