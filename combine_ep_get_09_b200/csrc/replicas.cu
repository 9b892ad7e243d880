// replicas.cu -- slots of busy experts spread over their redundant copies.
//
// DeepSeek's expert load balancer deploys extra copies of the experts in
// high demand (deepseekaiinsights, Open Source Week overview, "EPLB and
// DualPipe"); the page gives no rule for which copy a token uses.  Reading:
// the i-th slot of logical expert e, in the stable token-major order of the
// dispatch layout (i = slot_pos - off_e[e]), goes to copy i mod n_e, so the
// copies of one expert receive equal shares to within one slot.  The
// physical ids then go through the layout like any other ids.
#include "ep_internal.cuh"

namespace ep {
namespace {

constexpr int kRepThreads = 256;

template <typename IdT>
__global__ void __launch_bounds__(kRepThreads)
    map_replicas_kernel(const IdT *__restrict__ idx, long n, int E,
                        const int32_t *__restrict__ slot_pos, const int32_t *__restrict__ off_e,
                        const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_ids,
                        int32_t *__restrict__ phys, int32_t *d_err) {
  pdl_wait();
  for (long i = static_cast<long>(blockIdx.x) * kRepThreads + threadIdx.x; i < n;
       i += static_cast<long>(gridDim.x) * kRepThreads) {
    const long long e = static_cast<long long>(idx[i]);
    int out = -1;
    if (e >= 0 && e < E) {
      const int c0 = __ldg(rep_off + e), copies = __ldg(rep_off + e + 1) - c0;
      const int row = slot_pos[i];
      if (copies > 0 && row >= 0) {
        out = __ldg(rep_ids + c0 + (row - __ldg(off_e + e)) % copies);
      } else if (d_err != nullptr) {
        atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_INDEX);
      }
    } else if (e != -1 && d_err != nullptr) {
      atomicExch(reinterpret_cast<int *>(d_err), EP_ERR_INDEX);
    }
    phys[i] = out;
  }
}

}  // namespace

cudaError_t launch_map_replicas(const void *idx, bool int64_ids, int T, int k, int E,
                                const int32_t *slot_pos, const int32_t *off_e,
                                const int32_t *rep_off, const int32_t *rep_ids, int32_t *phys,
                                int32_t *d_err, cudaStream_t s, int *launches) {
  const long n = static_cast<long>(T) * k;
  if (n == 0) return cudaSuccess;
  ++*launches;
  if (int64_ids) {
    auto kern = map_replicas_kernel<long long>;
    const long grid = persistent_grid(reinterpret_cast<const void *>(kern), kRepThreads, 0,
                                      (n + 31) / 32, 0);
    return launch_pdl(kern, dim3(grid), dim3(kRepThreads), 0, s, 1,
                      static_cast<const long long *>(idx), n, E, slot_pos, off_e, rep_off,
                      rep_ids, phys, d_err);
  }
  auto kern = map_replicas_kernel<int32_t>;
  const long grid = persistent_grid(reinterpret_cast<const void *>(kern), kRepThreads, 0,
                                    (n + 31) / 32, 0);
  return launch_pdl(kern, dim3(grid), dim3(kRepThreads), 0, s, 1,
                    static_cast<const int32_t *>(idx), n, E, slot_pos, off_e, rep_off, rep_ids,
                    phys, d_err);
}

}  // namespace ep
