// Diagnostic kernel for the failure path of the bounded waits.
//
// One thread waits on an mbarrier that nothing arrives at.  After `limit` SM
// cycles the bounded wait records a timeout (bit 0 and wait site SITE_SELFTEST
// in bits 8..15 of the device error word) and the kernel returns: the path a
// broken pipeline takes, exercised without a fault, a trap or a hang.
#pragma once

#include "ptx.cuh"

namespace convrot {

constexpr unsigned SITE_SELFTEST = 15;

__global__ void __launch_bounds__(32) selftest_wait_timeout_kernel(long long limit) {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0u, &abort_word, SITE_SELFTEST, limit);
}

}  // namespace convrot
