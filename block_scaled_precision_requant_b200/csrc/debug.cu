// Test entry for the failure path: a kernel whose single pipeline wait can
// never be satisfied, so the bounded wait runs out, records its bit in the
// device status word and returns -- the same route a pipelined kernel takes
// when a peer role stops making progress.  Nothing faults or traps.
#include "common.cuh"
#include "kernels.h"

namespace bsr {

namespace {

__global__ void debug_wait_kernel(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0u, &abort_flag, status, DEV_ERR_TIMEOUT_DEBUG, limit_ns);
}

}  // namespace

cudaError_t launch_debug_wait(int* status, unsigned long long limit_ns, cudaStream_t stream) {
  debug_wait_kernel<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace bsr
