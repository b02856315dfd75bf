// selftest.cuh -- failure-detection self test for the bounded waits.
//
// One warp initialises an mbarrier that nothing will ever complete and waits
// on it with a short limit.  The wait gives up, records
// kStatusTimeoutTest in the status word and the kernel returns normally: no
// trap, no hang, the context stays usable.
#pragma once

#include "ptx.cuh"

namespace gqa {

__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(&bar, 0)) return;  // never completes
    if ((it & 63u) == 0 && global_timer_ns() - t0 > limit_ns) {
      report_status(kStatusTimeoutTest);
      return;
    }
  }
}

}  // namespace gqa
