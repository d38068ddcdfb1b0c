// Self-test of the device-side failure path: every wait of the library's kernels on an mbarrier
// gives up after kWaitTimeoutNs, records a code in the device error word and lets the kernel
// return, so that the context stays usable.  This kernel takes that path on purpose.
#include "common.cuh"
#include "internal.h"

namespace moss {

namespace {

// One thread waits on an mbarrier phase that nothing completes.
__global__ void wait_probe_kernel(unsigned* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, err, kErrSelfTest, &abort_flag);
  }
}

}  // namespace

cudaError_t launch_wait_probe(unsigned* err, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

}  // namespace moss
