// Failure-detection self-test. One CTA waits on an mbarrier that no thread ever completes, the
// situation of a pipeline wait whose producer has stopped. The wait is the library's own
// bounded wait (mbar_wait, the one every pipeline kernel uses): it gives up after timeout_ns of
// wall time, the kernel records MOE_DEVERR_WAIT_TIMEOUT in the error word and returns, and the
// context stays usable. Nothing faults, traps or spins without a bound.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

__global__ void wait_timeout_probe_kernel(int* err, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none ever comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns))
    record_error(err, MOE_DEVERR_WAIT_TIMEOUT);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(int* err, uint64_t timeout_ns, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(err, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
