// common.cuh -- shared pieces of the h3attn kernels: the device error word and
// bounded mbarrier waits.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace h3 {

// Error bits recorded by kernels in the device error word.
enum : uint32_t {
  kErrTimeout = 1u,       // a bounded wait gave up
  kErrBadBlockList = 2u,  // a block-sparse key list was not strictly ascending in range
  kErrBadSeqlens = 4u,    // a ragged launch's cu_seqlens broke its rules (the launch wrote nothing)
  kErrBounds = 8u,        // debug builds: a store index outside the launch's own extents (skipped)
};

// Device error word: [0] = sticky error bits, [1] = id of the last launch that
// failed (lets the other CTAs of that launch stop early without affecting later
// launches).  Lives in the library module (the library is one translation
// unit, so this is its only definition); read by h3attn_device_status().
__device__ uint32_t g_error_word[2];
// Where h3attn_device_status() has the error word exchanged for zero on the
// device, so that no error recorded between a read and a clear is lost.
__device__ uint32_t g_status_snapshot[2];

__global__ void status_exchange_kernel(int clear) {
  if (threadIdx.x == 0) {
    g_status_snapshot[0] = clear ? atomicExch(&g_error_word[0], 0u) : atomicOr(&g_error_word[0], 0u);
    g_status_snapshot[1] = clear ? atomicExch(&g_error_word[1], 0u) : atomicOr(&g_error_word[1], 0u);
  }
}

// Longest a thread waits on one barrier phase before declaring the launch failed.
constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s

struct LaunchCtl {
  uint32_t launch_id;  // distinct per host call, never 0
};

__device__ __forceinline__ bool launch_failed(const LaunchCtl& ctl) {
  return *reinterpret_cast<volatile uint32_t*>(&g_error_word[1]) == ctl.launch_id;
}

// An error that leaves the rest of the launch running (no launch id recorded).
__device__ __forceinline__ void report_error(uint32_t bits) { atomicOr(&g_error_word[0], bits); }

// Debug builds (compiled with H3ATTN_DEBUG_BOUNDS) check every global store's
// indices against the extents of the launch that makes it: an index outside them
// records kErrBounds and the store is skipped (no trap, nothing written out of
// place).  Release builds compile the check away.
#ifdef H3ATTN_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool store_in_bounds(bool in_bounds) {
  if (kDebugBounds && !in_bounds) {
    atomicOr(&g_error_word[0], kErrBounds);
    return false;
  }
  return true;
}

__device__ __forceinline__ void report_failure(const LaunchCtl& ctl, uint32_t bits) {
  atomicOr(&g_error_word[0], bits);
  atomicExch(&g_error_word[1], ctl.launch_id);
}

// Wait until the phase of `bar` with parity `parity` completes.  Returns false
// (and records a timeout) after kWaitLimitNs, or early if another CTA of this
// launch already failed.
// Each probe may suspend the thread for up to kSleepHintNs, so a waiting warp
// neither spins nor takes issue slots from the warps doing the work.
constexpr uint32_t kSleepHintNs = 1000000;  // 1 ms

__device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, LaunchCtl ctl) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (ptx::mbar_test_sleep(bar, parity, kSleepHintNs)) return true;
    if ((it & 15u) == 0) {
      if (launch_failed(ctl)) return false;
      if (ptx::globaltimer_ns() - t0 > kWaitLimitNs) {
        report_failure(ctl, kErrTimeout);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const LaunchCtl& ctl) {
  if (ptx::mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ctl);
}

// Bounded wait that ignores the launch-failed flag (used on the way out of a
// failed launch, to drain copies and tensor-core operations still in flight).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = ptx::globaltimer_ns();
  while (!ptx::mbar_test(bar, parity)) {
    if (ptx::globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// How long a thread leaving a failed launch waits for its own operations in flight.
constexpr uint64_t kDrainLimitNs = 20000000ull;  // 20 ms

}  // namespace h3
