// Self-test of the bounded waits every pipelined kernel relies on.
//
// One CTA waits on a shared-memory mbarrier that nothing ever signals, with
// the same mbar_wait the decode and extend kernels use.  The wait gives up
// after about one second, the kernel records PKV_DEV_ERR_TIMEOUT in the
// caller's error word and returns, and the context stays usable.  Nothing
// here faults, traps or spins without bound.
#include "common.cuh"
#include "launch.h"

namespace pkv {

namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait(&bar, 0);  // no arrival will ever come
  if (!ok && threadIdx.x == 0) set_err(err, PKV_DEV_ERR_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout(int32_t* err, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(err);
  return cudaGetLastError();
}

}  // namespace pkv
