// Self-test of the bounded waits (fb_selftest_wait_timeout): the failure path the
// attention kernels take when an asynchronous copy never completes, exercised
// without any fault -- the wait runs out, the status word records it, the
// kernel returns.
#pragma once

#include "fb_kernels.cuh"

namespace fb {

// A wait that nothing satisfies: mbar_wait gives up after kWaitLimitNs.
__global__ void wait_timeout_selftest_kernel() {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait(&bar, 0)) record_status(kDevTimeout);
  }
}

}  // namespace fb
