// diag.cu -- a check of the bounded-wait failure path that every kernel of this library
// uses (hy_common.cuh, mbar_wait): one thread waits on an mbarrier that nothing arrives
// on; the wait gives up after its limit, records HYMBA_ERR_TIMEOUT in the status word and
// the kernel returns, so the GPU context stays usable.
#include "hy_common.cuh"
#include "hy_kernels.h"
#include "hymba.h"

namespace hy {
namespace {

__global__ void __launch_bounds__(32) wait_nothing_kernel(unsigned* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status, &abort_flag, limit_ns);
}

}  // namespace
}  // namespace hy

extern "C" hymba_status_t hymba_check_wait_timeout(void* workspace, size_t ws_bytes, unsigned limit_us,
                                                   void* stream) {
  if (!workspace || ws_bytes < 256) return HYMBA_ERR_WORKSPACE;
  if (limit_us < 1 || limit_us > 1000000) return HYMBA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* status = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(unsigned), st) != cudaSuccess) return HYMBA_ERR_CUDA;
  hy::wait_nothing_kernel<<<1, 32, 0, st>>>(status, 1000ull * limit_us);
  return cudaGetLastError() == cudaSuccess ? HYMBA_OK : HYMBA_ERR_CUDA;
}
