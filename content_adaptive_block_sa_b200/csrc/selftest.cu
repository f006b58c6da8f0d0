// Device self-test of the failure path, with no fault: every CTA waits on an
// mbarrier that no thread arrives at, through the bounded wait every kernel of
// the library uses (its 4 s wall-time limit included). The first CTA to give
// up records SA_ERR_TIMEOUT at location kSelftestWhere in the status word; the
// others leave on seeing the word. Nothing traps, and the context stays usable.
#include "sa_common.cuh"
#include "sm100.cuh"

namespace sa {

constexpr int kSelftestWhere = 900;

__global__ void __launch_bounds__(32) wait_timeout_kernel(DeviceStatus* st) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    abort_flag = 0;
    sm100::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    sm100::mbar_wait(&bar, 0, &abort_flag, st, kSelftestWhere);  // nobody arrives
}

cudaError_t launch_wait_timeout_selftest(void* ws, int n_ctas, cudaStream_t s) {
  wait_timeout_kernel<<<n_ctas, 32, 0, s>>>(static_cast<DeviceStatus*>(ws));
  return cudaGetLastError();
}

}  // namespace sa
