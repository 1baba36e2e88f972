// Bounded mbarrier waits and ring positions shared by the persistent tcgen05 kernels of the
// comparison paths (materialised scores, full-rank router).
#pragma once
#include "more_internal.cuh"
#include "sm100_ptx.cuh"

namespace more {
namespace sm100 {

constexpr uint64_t kWaitLimitNs = 4000000000ull;

// Slow path of the bounded wait: false once kWaitLimitNs pass (the device error word records
// MORE_DEVERR_WAIT_TIMEOUT and the abort flag stops the CTA's other roles) or once another
// thread of the CTA has raised the abort flag.
__device__ __noinline__ inline bool bounded_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                      unsigned int* status) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait_sleep(bar, parity, 200000u)) return true;
    if ((spin & 3u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        atomicOr(status, MORE_DEVERR_WAIT_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// The first attempt suspends in hardware until the phase completes (or ~65 us pass), so a
// normal wait is one instruction and the bounded loop is a rare call.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                             unsigned int* status) {
  if (mbar_try_wait_sleep(bar, parity, 65536u)) return true;
  return bounded_wait_slow(bar, parity, abort_flag, status);
}

// Position of one thread in a ring of mbarrier-guarded buffers.
struct RingPos {
  int i = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void next(int n) {
    if (++i == n) {
      i = 0;
      phase ^= 1u;
    }
  }
};

}  // namespace sm100
}  // namespace more
