// Device self-test of the failure path, with no fault: every CTA waits on an
// mbarrier that no thread arrives at, through the bounded wait every kernel of
// the library uses (its 4 s wall-time limit included). The first CTA to give
// up records SA_ERR_TIMEOUT at location kSelftestWhere in the status word; the
// others leave on seeing the word. Nothing traps, and the context stays usable.
#include "sa_common.cuh"
#include "sa_selftest.h"
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

}  // namespace sa

extern "C" sa_status sa_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t n_ctas,
                                              sa_stream_t stream) {
  if (n_ctas < 1 || n_ctas > 1024 || ws == nullptr) return SA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return SA_ERR_INVALID_ARG;
  if (ws_bytes < sa::kStatusBytes) return SA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaMemsetAsync(ws, 0, sa::kStatusBytes, s) != cudaSuccess) return SA_ERR_CUDA;
  sa::wait_timeout_kernel<<<n_ctas, 32, 0, s>>>(static_cast<sa::DeviceStatus*>(ws));
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
