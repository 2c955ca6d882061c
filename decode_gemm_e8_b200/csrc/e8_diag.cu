// Diagnostic kernel for the failure-detection path: one thread waits on an
// mbarrier that nothing will ever complete, gives up after `limit_ns`, and
// reports through the device status word exactly like the pipeline kernels'
// bounded waits do.  It touches no memory but its own shared barrier and the
// status word, so the context stays usable.
#include "e8_common.cuh"
#include "e8_internal.h"

namespace e8 {

__global__ void k_wait_never_signalled(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(&bar, 0)) {
    if (global_timer_ns() - t0 > limit_ns) {
      atomicOr(status, kDevTimeoutFull);
      return;
    }
  }
}

cudaError_t launch_wait_never_signalled(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  k_wait_never_signalled<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace e8
