// Self-test of the bounded pipeline wait: one thread waits on an mbarrier that
// nothing arrives at.  The wait gives up after its limit (1 s of %globaltimer)
// and records MOE_ERR_TIMEOUT in the status word, the path every tcgen05 kernel
// of the library takes when a TMA or MMA completion never arrives; the kernel
// then returns normally, so the context stays usable.
#include "common.cuh"
#include "kernels.h"

namespace moe {

__global__ void k_selftest_bounded_wait(int* status) {
  pdl_wait_and_trigger();
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_s = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_s, status);  // no arrival: returns false after the limit
  }
}

cudaError_t launch_selftest_bounded_wait(int* status, cudaStream_t s) {
  return launch_kernel(k_selftest_bounded_wait, dim3(1), dim3(32), 0, s, 1, status);
}

}  // namespace moe
