// Self-test of the bounded device waits that every kernel of the library uses
// (sm100.cuh, mbar_wait): one thread waits on an mbarrier that nothing arrives
// at.  The wait gives up after its wall-clock budget, records a code in the
// layer's device error word and returns, so the kernel ends and the context
// stays usable; svdq_check then reports SVDQ_ETIMEOUT.  This exercises the
// failure-detection path without a fault, a trap or a hang.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100.cuh"

namespace svdq {

namespace {

__global__ void __launch_bounds__(32, 1) wait_selftest_kernel(int* err, unsigned long long budget_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    dev::mbar_init(&bar, 1);
    abort_flag = 0;
    dev::fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !dev::mbar_wait(&bar, 0, &abort_flag, budget_ns)) atomicCAS(err, 0, 0x3ff);
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, unsigned long long budget_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(err, budget_ns);
  return cudaGetLastError();
}

}  // namespace svdq
