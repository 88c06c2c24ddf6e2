// Bounded mbarrier waits shared by the persistent kernels.  A wait that runs past its
// limit records kStatusTimeout in the device status word and raises the CTA's abort
// flag; the kernel then lets its in-flight copies land and returns.
#pragma once
#include "internal.cuh"
#include "ptx.cuh"

namespace bitmoe {
namespace {

constexpr long long kDrainNs = 500000000LL;  // bound on draining in-flight work

// Bounded wait by one thread; false if the limit ran out or another role aborted.  The
// loop is try_wait alone (which itself parks the thread for a short, hardware-chosen
// time); the abort flag and the clock are read only every 64 tries, so waiting threads
// add little shared-memory traffic.  (Limits under 100 us are checked on every try.)
__device__ bool wait_one(uint32_t bar, uint32_t parity, long long limit, volatile int* abort_flag,
                         int* status) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  const uint32_t every = limit < 100000 ? 0u : 63u;
  for (uint32_t i = 1;; ++i) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if ((i & every) == 0) {
      if (*abort_flag) return false;
      if ((long long)(ptx::globaltimer() - t0) > limit) {
        *abort_flag = 1;
        atomicOr(status, kStatusTimeout);
        return false;
      }
    }
  }
}
// Same, decided by lane 0 and shared with the whole warp (keeps the warp converged).
__device__ __forceinline__ bool wait_warp(uint32_t bar, uint32_t parity, long long limit,
                                          volatile int* abort_flag, int* status) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_one(bar, parity, limit, abort_flag, status) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}
// Wait for in-flight work to land during teardown (ignores the abort flag).
__device__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait(bar, parity)) {
    if ((long long)(ptx::globaltimer() - t0) > kDrainNs) break;
  }
}

}  // namespace
}  // namespace bitmoe
