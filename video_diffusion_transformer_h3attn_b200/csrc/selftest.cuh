// selftest.cuh -- failure-detection self-test of the bounded barrier waits that
// every h3attn kernel uses (h3attn_selftest_wait_timeout).
#pragma once

#include <cstdint>

#include "common.cuh"

namespace h3 {

// Self-test of the bounded wait: one thread waits for the first phase of a
// barrier that expects one arrival and never gets it.  The wait gives up after
// kWaitLimitNs and records kErrTimeout.
__global__ void wait_timeout_selftest_kernel(LaunchCtl ctl) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbarrier_init();
  mbar_wait(b, 0u, ctl);
}

}  // namespace h3
