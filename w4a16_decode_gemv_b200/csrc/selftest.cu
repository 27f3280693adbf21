// Diagnostics for the bounded waits: a kernel whose barrier wait runs out.
//
// Every wait of the GEMM kernels on an mbarrier is bounded by the device clock;
// when one gives up, the kernel sets kDevWaitTimeout in the workspace status
// word, lets its copies in flight land and returns, and w4a16_gemm_check
// reports W4A16_ERR_DEVICE.  This kernel takes the same steps on a barrier that
// nothing ever completes, so that the path can be exercised without a fault.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_probe(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected; none is made
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t t0 = globaltimer_ns();
  bool done = mbar_try_wait(&bar, 0u);
  while (!done && globaltimer_ns() - t0 <= limit_ns) done = mbar_try_wait(&bar, 0u);
  if (!done && threadIdx.x == 0) atomicOr(status, kDevWaitTimeout);
}

}  // namespace

cudaError_t launch_wait_timeout_probe(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  wait_timeout_probe<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace w4a16
