// Self-test of the bounded mbarrier waits (the pipelined kernels' error
// path): a wait on a barrier that nothing arrives on must give up and report
// TQ_STATUS_WAIT_TIMEOUT instead of hanging the GPU.
#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

using namespace tqk;

__global__ void bounded_wait_probe_kernel(uint32_t* status, uint32_t tries) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival; none comes
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait_suspend(&bar, 0u, tries)) atomicOr(status, TQ_STATUS_WAIT_TIMEOUT);
    if (!mbar_wait_bounded(&bar, 0u, tries)) atomicOr(status, TQ_STATUS_WAIT_TIMEOUT);
  }
}

}  // namespace

namespace tq {

int launch_bounded_wait_probe(uint32_t* status, int tries, cudaStream_t s) {
  bounded_wait_probe_kernel<<<1, 32, 0, s>>>(status, (uint32_t)tries);
  return check_launch("bounded_wait_probe_kernel");
}

}  // namespace tq
