// ep_abi.cu -- the extern "C" entry points of libep.so: argument checks,
// launch, error reporting.  Every check happens before anything is
// enqueued; the kernels live in layout.cu, layout_dispatch.cu,
// dispatch_bf16.cu, dispatch_fp8.cu, combine.cu, pad_layout.cu and
// replicas.cu.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include "bulk.cuh"
#include "ep_internal.cuh"

namespace {

thread_local char g_err[512] = "";
std::atomic<uint64_t> g_launches{0};

ep_status_t fail(ep_status_t st, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

ep_status_t from_cuda(cudaError_t e, const char *where) {
  if (e == cudaSuccess) return EP_OK;
  return fail(EP_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorString(e),
              cudaGetErrorName(e));
}

bool aligned(const void *p, size_t a) {
  return reinterpret_cast<uintptr_t>(p) % a == 0;
}

// Shared size checks of dispatch and combine.
ep_status_t check_rows(const char *fn, int T, int H, int k, int num_sms) {
  if (T < 0) return fail(EP_ERR_INVALID_ARG, "%s: T=%d < 0", fn, T);
  if (H <= 0) return fail(EP_ERR_INVALID_ARG, "%s: H=%d <= 0", fn, H);
  if (k < 1) return fail(EP_ERR_INVALID_ARG, "%s: k=%d < 1", fn, k);
  if (num_sms < 0) return fail(EP_ERR_INVALID_ARG, "%s: num_sms=%d < 0", fn, num_sms);
  if (k > EP_MAX_K)
    return fail(EP_ERR_UNSUPPORTED, "%s: k=%d > %d", fn, k, EP_MAX_K);
  if (H % 8 != 0)
    return fail(EP_ERR_UNSUPPORTED, "%s: H=%d is not a multiple of 8", fn, H);
  if (static_cast<long long>(T) * k > 0x7fffffffLL)
    return fail(EP_ERR_UNSUPPORTED, "%s: T*k=%lld does not fit int32", fn,
                static_cast<long long>(T) * k);
  return EP_OK;
}

#define EP_REQUIRE_PTR(fn, p, align)                                          \
  do {                                                                        \
    if ((p) == nullptr)                                                       \
      return fail(EP_ERR_INVALID_ARG, "%s: %s is NULL", fn, #p);              \
    if (!aligned((p), (align)))                                               \
      return fail(EP_ERR_INVALID_ARG, "%s: %s is not %d-byte aligned", fn, #p, \
                  static_cast<int>(align));                                   \
  } while (0)

}  // namespace

namespace ep {

ep_status_t record_error(ep_status_t status, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return status;
}

int device_sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
    n = 1;
  if (dev < 64) cached[dev] = n;
  return n;
}

int max_dynamic_smem(const void *kernel) {
  static std::mutex mu;
  static std::map<std::pair<int, const void *>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 48 << 10;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find({dev, kernel});
  if (it != cache.end()) return it->second;
  int optin = 48 << 10;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
      cudaSuccess)
    optin = 48 << 10;
  cudaFuncAttributes fa = {};
  const int stat =
      cudaFuncGetAttributes(&fa, kernel) == cudaSuccess ? static_cast<int>(fa.sharedSizeBytes)
                                                        : 1024;
  const int n = optin - stat;
  cache[{dev, kernel}] = n;
  return n;
}

long persistent_grid(const void *kernel, int threads, int smem_bytes, long warp_items,
                     int num_sms) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void *, int, int>, int> cache;
  int dev = 0;
  cudaGetDevice(&dev);
  int per_sm = 0;
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(dev, kernel, threads, smem_bytes);
    auto it = cache.find(key);
    if (it != cache.end()) {
      per_sm = it->second;
    } else {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem_bytes) !=
              cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      cache[key] = per_sm;
    }
  }
  const int sms = num_sms > 0 ? num_sms : device_sm_count();
  const long warps_per_block = threads / kWarp;
  const long need = (warp_items + warps_per_block - 1) / warps_per_block;
  const long cap = static_cast<long>(sms) * per_sm;
  return need < cap ? need : cap;
}

namespace {
std::atomic<int> g_first_wait_polls{kMaxBarrierPolls};
}  // namespace

int first_wait_polls() { return g_first_wait_polls.load(std::memory_order_relaxed); }

cudaError_t raise_dynamic_smem(const void *kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<int, const void *>, int> done;
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find({dev, kernel});
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err == cudaSuccess) done[{dev, kernel}] = bytes;
  return err;
}

}  // namespace ep

extern "C" {

int ep_abi_version(void) { return 5; }

const char *ep_last_error_string(void) { return g_err; }

uint64_t ep_kernel_launches(void) { return g_launches.load(); }

void ep_debug_expire_first_wait(int on) {
  ep::g_first_wait_polls.store(on ? 0 : ep::kMaxBarrierPolls, std::memory_order_relaxed);
}

static ep_status_t check_layout_sizes(const char *fn, int T, int k, int E, int R) {
  if (T < 0) return fail(EP_ERR_INVALID_ARG, "%s: T=%d < 0", fn, T);
  if (k < 1) return fail(EP_ERR_INVALID_ARG, "%s: k=%d < 1", fn, k);
  if (E < 1) return fail(EP_ERR_INVALID_ARG, "%s: E=%d < 1", fn, E);
  if (R < 1) return fail(EP_ERR_INVALID_ARG, "%s: R=%d < 1", fn, R);
  if (E % R != 0)
    return fail(EP_ERR_INVALID_ARG, "%s: E=%d is not a multiple of R=%d", fn, E, R);
  if (k > E) return fail(EP_ERR_INVALID_ARG, "%s: k=%d > E=%d", fn, k, E);
  if (k > EP_MAX_K) return fail(EP_ERR_UNSUPPORTED, "%s: k=%d > %d", fn, k, EP_MAX_K);
  if (E > EP_MAX_E) return fail(EP_ERR_UNSUPPORTED, "%s: E=%d > %d", fn, E, EP_MAX_E);
  if (R > EP_MAX_R) return fail(EP_ERR_UNSUPPORTED, "%s: R=%d > %d", fn, R, EP_MAX_R);
  if (static_cast<long long>(T) * k > 0x7fffffffLL)
    return fail(EP_ERR_UNSUPPORTED, "%s: T*k does not fit int32", fn);
  return EP_OK;
}

static ep::LayoutArgs expert_layout_args(const void *idx, int idx_is_int64, int T, int k, int E,
                                        int R, int32_t *cnt_e, int32_t *cnt_r,
                                        uint8_t *in_rank, int32_t *off_e, int32_t *off_r,
                                        int32_t *slot_pos, int32_t *recv_src, void *ws,
                                        int32_t *d_err) {
  ep::LayoutArgs a{};
  a.idx = idx;
  a.id_kind = idx_is_int64 ? ep::kIdsInt64 : ep::kIdsInt32;
  a.T = T;
  a.k = k;
  a.E = E;
  a.R = R;
  a.cnt_e = cnt_e;
  a.cnt_r = cnt_r;
  a.off_e = off_e;
  a.off_r = off_r;
  a.slot_pos = slot_pos;
  a.recv_src = recv_src;
  a.in_rank = in_rank;
  a.ws = ws;
  a.d_err = d_err;
  return a;
}

size_t ep_layout_workspace_bytes(int T, int k, int E, int R) {
  if (check_layout_sizes("ep_layout_workspace_bytes", T, k, E, R) != EP_OK) return 0;
  return ep::layout_workspace_bytes(T, k, E, R);
}

ep_status_t ep_get_layout(const void *idx, int idx_is_int64, int T, int k,
                          int E, int R, int32_t *cnt_e, int32_t *cnt_r,
                          uint8_t *in_rank, int32_t *off_e, int32_t *off_r,
                          int32_t *slot_pos, int32_t *recv_src, void *ws,
                          size_t ws_bytes, int32_t *d_err, void *stream) {
  static const char fn[] = "ep_get_layout";
  g_err[0] = '\0';
  ep_status_t st = check_layout_sizes(fn, T, k, E, R);
  if (st != EP_OK) return st;
  EP_REQUIRE_PTR(fn, cnt_e, 4);
  EP_REQUIRE_PTR(fn, cnt_r, 4);
  EP_REQUIRE_PTR(fn, off_e, 4);
  EP_REQUIRE_PTR(fn, off_r, 4);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, idx, idx_is_int64 ? 8 : 4);
    EP_REQUIRE_PTR(fn, in_rank, 1);
    EP_REQUIRE_PTR(fn, slot_pos, 4);
    EP_REQUIRE_PTR(fn, recv_src, 4);
  }
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  const size_t need = ep::layout_workspace_bytes(T, k, E, R);
  if (need > 0) {
    EP_REQUIRE_PTR(fn, ws, 16);
    if (ws_bytes < need)
      return fail(EP_ERR_INVALID_ARG, "%s: ws_bytes=%zu < %zu needed", fn, ws_bytes, need);
  }
  const ep::LayoutArgs a = expert_layout_args(idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r,
                                               in_rank, off_e, off_r, slot_pos, recv_src, ws,
                                               d_err);
  int n = 0;
  const cudaError_t e = ep::launch_layout(a, static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

size_t ep_rank_layout_workspace_bytes(int T, int R) {
  if (T < 0 || R < 1 || R > EP_MAX_R || static_cast<long long>(T) * R > 0x7fffffffLL) return 0;
  return ep::layout_workspace_bytes(T, R, R, 1);
}

ep_status_t ep_get_rank_layout(const uint8_t *in_rank, int T, int R, int32_t *cnt_r,
                               int32_t *off_r, int32_t *rank_row, int32_t *rank_src,
                               void *ws, size_t ws_bytes, void *stream) {
  static const char fn[] = "ep_get_rank_layout";
  g_err[0] = '\0';
  if (T < 0) return fail(EP_ERR_INVALID_ARG, "%s: T=%d < 0", fn, T);
  if (R < 1) return fail(EP_ERR_INVALID_ARG, "%s: R=%d < 1", fn, R);
  if (R > EP_MAX_R) return fail(EP_ERR_UNSUPPORTED, "%s: R=%d > %d", fn, R, EP_MAX_R);
  if (static_cast<long long>(T) * R > 0x7fffffffLL)
    return fail(EP_ERR_UNSUPPORTED, "%s: T*R does not fit int32", fn);
  EP_REQUIRE_PTR(fn, cnt_r, 4);
  EP_REQUIRE_PTR(fn, off_r, 4);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, in_rank, 1);
    EP_REQUIRE_PTR(fn, rank_row, 4);
    EP_REQUIRE_PTR(fn, rank_src, 4);
  }
  const size_t need = ep::layout_workspace_bytes(T, R, R, 1);
  if (need > 0) {
    EP_REQUIRE_PTR(fn, ws, 16);
    if (ws_bytes < need)
      return fail(EP_ERR_INVALID_ARG, "%s: ws_bytes=%zu < %zu needed", fn, ws_bytes, need);
  }
  // the expert layout of the mask: slot (t, r) "chooses expert r" when token
  // t is in rank r; experts = ranks, one group holding them all
  ep::LayoutArgs a{};
  a.idx = in_rank;
  a.id_kind = ep::kIdsMask;
  a.T = T;
  a.k = R;
  a.E = R;
  a.R = 1;
  a.cnt_e = cnt_r;
  a.off_e = off_r;
  a.slot_pos = rank_row;
  a.recv_src = rank_src;
  a.ws = ws;
  int n = 0;
  const cudaError_t e = ep::launch_layout(a, static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

// Rows of a receive buffer: recv_rows, or T*k when it is 0.
static ep_status_t receive_rows(const char *fn, int recv_rows, int T, int k, long *n_rows) {
  if (recv_rows < 0) return fail(EP_ERR_INVALID_ARG, "%s: recv_rows=%d < 0", fn, recv_rows);
  *n_rows = recv_rows > 0 ? recv_rows : static_cast<long>(T) * k;
  return EP_OK;
}

ep_status_t ep_dispatch(const void *x, int T, int H, int k,
                        const int32_t *slot_pos, int fp8, void *recv,
                        float *recv_scale, int recv_rows, int num_sms, int32_t *d_err,
                        void *stream) {
  static const char fn[] = "ep_dispatch";
  g_err[0] = '\0';
  ep_status_t st = check_rows(fn, T, H, k, num_sms);
  if (st != EP_OK) return st;
  long n_rows = 0;
  st = receive_rows(fn, recv_rows, T, k, &n_rows);
  if (st != EP_OK) return st;
  if (fp8 && H % 128 != 0)
    return fail(EP_ERR_UNSUPPORTED, "%s: fp8 needs H %% 128 == 0 (H=%d)", fn, H);
  if (T == 0) return EP_OK;
  EP_REQUIRE_PTR(fn, x, 16);
  EP_REQUIRE_PTR(fn, slot_pos, 4);
  EP_REQUIRE_PTR(fn, recv, 16);
  if (fp8) EP_REQUIRE_PTR(fn, recv_scale, 4);
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  int n = 0;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      fp8 ? ep::launch_dispatch_fp8(x, T, H, k, slot_pos, recv, recv_scale, n_rows, num_sms,
                                    d_err, s, &n)
          : ep::launch_dispatch_bf16(x, T, H, k, slot_pos, recv, n_rows, num_sms, d_err, s, &n);
  g_launches += n;
  return from_cuda(e, fn);
}

ep_status_t ep_layout_dispatch(const void *idx, int idx_is_int64, int T, int k, int E, int R,
                               const void *x, int H, int fp8, int32_t *cnt_e, int32_t *cnt_r,
                               uint8_t *in_rank, int32_t *off_e, int32_t *off_r,
                               int32_t *slot_pos, int32_t *recv_src, void *recv,
                               float *recv_scale, void *ws, size_t ws_bytes, int num_sms,
                               int32_t *d_err, void *stream) {
  static const char fn[] = "ep_layout_dispatch";
  ep_status_t st = ep::check_layout_args(fn, idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r,
                                         in_rank, off_e, off_r, slot_pos, recv_src, d_err);
  if (st != EP_OK) return st;
  st = check_rows(fn, T, H, k, num_sms);
  if (st != EP_OK) return st;
  if (fp8 && H % 128 != 0)
    return fail(EP_ERR_UNSUPPORTED, "%s: fp8 needs H %% 128 == 0 (H=%d)", fn, H);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, x, 16);
    EP_REQUIRE_PTR(fn, recv, 16);
    if (fp8) EP_REQUIRE_PTR(fn, recv_scale, 4);
  }
  const size_t need = ep::layout_workspace_bytes(T, k, E, R);
  if (need > 0) {
    EP_REQUIRE_PTR(fn, ws, 16);
    if (ws_bytes < need)
      return fail(EP_ERR_INVALID_ARG, "%s: ws_bytes=%zu < %zu needed", fn, ws_bytes, need);
  }
  const ep::LayoutArgs a = expert_layout_args(idx, idx_is_int64, T, k, E, R, cnt_e, cnt_r,
                                               in_rank, off_e, off_r, slot_pos, recv_src, ws,
                                               d_err);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  int n = 0;
  cudaError_t e;
  if (ep::layout_dispatch_fusable(T, k, E, R, H, fp8 != 0, recv_scale)) {
    e = ep::launch_layout_dispatch(a, x, H, fp8 != 0, recv, recv_scale, num_sms, s, &n);
  } else {
    e = ep::launch_layout(a, s, &n);
    if (e == cudaSuccess)
      e = fp8 ? ep::launch_dispatch_fp8(x, T, H, k, slot_pos, recv, recv_scale,
                                        static_cast<long>(T) * k, num_sms, d_err, s, &n)
              : ep::launch_dispatch_bf16(x, T, H, k, slot_pos, recv, static_cast<long>(T) * k,
                                         num_sms, d_err, s, &n);
  }
  g_launches += n;
  return from_cuda(e, fn);
}

ep_status_t ep_combine(const void *y, int y_rows, int T, int H, int k,
                       const int32_t *slot_pos, const float *w, void *out,
                       int num_sms, int32_t *d_err, void *stream) {
  static const char fn[] = "ep_combine";
  g_err[0] = '\0';
  ep_status_t st = check_rows(fn, T, H, k, num_sms);
  if (st != EP_OK) return st;
  long n_rows = 0;
  st = receive_rows(fn, y_rows, T, k, &n_rows);
  if (st != EP_OK) return st;
  if (T == 0) return EP_OK;
  EP_REQUIRE_PTR(fn, y, 16);
  EP_REQUIRE_PTR(fn, slot_pos, 4);
  if (w != nullptr && !aligned(w, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: w is not 4-byte aligned", fn);
  EP_REQUIRE_PTR(fn, out, 16);
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  int n = 0;
  const cudaError_t e = ep::launch_combine(y, n_rows, T, H, k, slot_pos, w, out, num_sms, d_err,
                                           static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

ep_status_t ep_combine_fp8(const void *y_q, const float *y_scale, int y_rows, int T, int H,
                           int k, const int32_t *slot_pos, const float *w, void *out,
                           int num_sms, int32_t *d_err, void *stream) {
  static const char fn[] = "ep_combine_fp8";
  g_err[0] = '\0';
  ep_status_t st = check_rows(fn, T, H, k, num_sms);
  if (st != EP_OK) return st;
  if (H % 128 != 0)
    return fail(EP_ERR_UNSUPPORTED, "%s: H=%d is not a multiple of 128", fn, H);
  long n_rows = 0;
  st = receive_rows(fn, y_rows, T, k, &n_rows);
  if (st != EP_OK) return st;
  if (T == 0) return EP_OK;
  EP_REQUIRE_PTR(fn, y_q, 16);
  EP_REQUIRE_PTR(fn, y_scale, 4);
  EP_REQUIRE_PTR(fn, slot_pos, 4);
  if (w != nullptr && !aligned(w, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: w is not 4-byte aligned", fn);
  EP_REQUIRE_PTR(fn, out, 16);
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  int n = 0;
  const cudaError_t e =
      ep::launch_combine_fp8(y_q, y_scale, n_rows, T, H, k, slot_pos, w, out, num_sms, d_err,
                             static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

ep_status_t ep_map_replicas(const void *idx, int idx_is_int64, int T, int k, int E,
                            const int32_t *slot_pos, const int32_t *off_e,
                            const int32_t *rep_off, const int32_t *rep_ids, int32_t *phys_idx,
                            int32_t *d_err, void *stream) {
  static const char fn[] = "ep_map_replicas";
  g_err[0] = '\0';
  if (T < 0) return fail(EP_ERR_INVALID_ARG, "%s: T=%d < 0", fn, T);
  if (k < 1) return fail(EP_ERR_INVALID_ARG, "%s: k=%d < 1", fn, k);
  if (E < 1) return fail(EP_ERR_INVALID_ARG, "%s: E=%d < 1", fn, E);
  if (static_cast<long long>(T) * k > 0x7fffffffLL)
    return fail(EP_ERR_UNSUPPORTED, "%s: T*k does not fit int32", fn);
  EP_REQUIRE_PTR(fn, off_e, 4);
  EP_REQUIRE_PTR(fn, rep_off, 4);
  EP_REQUIRE_PTR(fn, rep_ids, 4);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, idx, idx_is_int64 ? 8 : 4);
    EP_REQUIRE_PTR(fn, slot_pos, 4);
    EP_REQUIRE_PTR(fn, phys_idx, 4);
  }
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  int n = 0;
  const cudaError_t e =
      ep::launch_map_replicas(idx, idx_is_int64 != 0, T, k, E, slot_pos, off_e, rep_off,
                              rep_ids, phys_idx, d_err, static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

size_t ep_aligned_rows(int T, int k, int E, int align) {
  if (T < 0 || k < 1 || E < 1 || align < 1) return 0;
  const long long rows = static_cast<long long>(T) * k + static_cast<long long>(E) * (align - 1);
  return rows > 0x7fffffffLL ? 0 : static_cast<size_t>(rows);
}

ep_status_t ep_pad_layout(const int32_t *cnt_e, const int32_t *slot_pos, int T, int k, int E,
                          int align, int32_t *off_pad, int32_t *slot_pos_pad,
                          int32_t *recv_src_pad, void *stream) {
  static const char fn[] = "ep_pad_layout";
  g_err[0] = '\0';
  if (T < 0) return fail(EP_ERR_INVALID_ARG, "%s: T=%d < 0", fn, T);
  if (k < 1) return fail(EP_ERR_INVALID_ARG, "%s: k=%d < 1", fn, k);
  if (E < 1) return fail(EP_ERR_INVALID_ARG, "%s: E=%d < 1", fn, E);
  if (align < 1) return fail(EP_ERR_INVALID_ARG, "%s: align=%d < 1", fn, align);
  if (E > EP_MAX_E) return fail(EP_ERR_UNSUPPORTED, "%s: E=%d > %d", fn, E, EP_MAX_E);
  if (ep_aligned_rows(T, k, E, align) == 0 && T > 0)
    return fail(EP_ERR_UNSUPPORTED, "%s: T*k + E*(align-1) does not fit int32", fn);
  EP_REQUIRE_PTR(fn, cnt_e, 4);
  EP_REQUIRE_PTR(fn, off_pad, 4);
  EP_REQUIRE_PTR(fn, recv_src_pad, 4);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, slot_pos, 4);
    EP_REQUIRE_PTR(fn, slot_pos_pad, 4);
  }
  int n = 0;
  const cudaError_t e = ep::launch_pad_layout(cnt_e, slot_pos, T, k, E, align, off_pad,
                                              slot_pos_pad, recv_src_pad,
                                              static_cast<cudaStream_t>(stream), &n);
  g_launches += n;
  return from_cuda(e, fn);
}

ep_status_t ep_read_error(const int32_t *d_err, void *stream) {
  static const char fn[] = "ep_read_error";
  g_err[0] = '\0';
  EP_REQUIRE_PTR(fn, d_err, 4);
  int32_t h = 0;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, d_err, sizeof h, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return from_cuda(e, fn);
  return h;
}

}  // extern "C"

namespace ep {

// The argument checks of ep_get_layout minus the workspace, for entry
// points that supply their own scratch.
ep_status_t check_layout_args(const char *fn, const void *idx, int idx_is_int64, int T,
                              int k, int E, int R, const int32_t *cnt_e,
                              const int32_t *cnt_r, const uint8_t *in_rank,
                              const int32_t *off_e, const int32_t *off_r,
                              const int32_t *slot_pos, const int32_t *recv_src,
                              const int32_t *d_err) {
  g_err[0] = '\0';
  ep_status_t st = check_layout_sizes(fn, T, k, E, R);
  if (st != EP_OK) return st;
  EP_REQUIRE_PTR(fn, cnt_e, 4);
  EP_REQUIRE_PTR(fn, cnt_r, 4);
  EP_REQUIRE_PTR(fn, off_e, 4);
  EP_REQUIRE_PTR(fn, off_r, 4);
  if (T > 0) {
    EP_REQUIRE_PTR(fn, idx, idx_is_int64 ? 8 : 4);
    EP_REQUIRE_PTR(fn, in_rank, 1);
    EP_REQUIRE_PTR(fn, slot_pos, 4);
    EP_REQUIRE_PTR(fn, recv_src, 4);
  }
  if (d_err != nullptr && !aligned(d_err, 4))
    return fail(EP_ERR_INVALID_ARG, "%s: d_err is not 4-byte aligned", fn);
  return EP_OK;
}

}  // namespace ep
