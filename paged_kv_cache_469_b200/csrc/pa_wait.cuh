// pa_wait.cuh -- time-bounded waits shared by the kernels of libpa.so.
//
// No wait in this library may hang a GPU.  Every wait on work of another warp
// of the same CTA -- an mbarrier phase (a TMA copy, an MMA, another role's
// arrival) or a flag in shared memory -- gives up after a time limit read from
// %globaltimer.  The warp that gives up records kStatusWaitTimeout in the
// workspace status word and raises the CTA's abort flag; every other waiting
// role of the CTA sees the flag and returns false as well, so the whole CTA
// winds down and the context stays usable.  A timeout means a library bug or a
// GPU fault, never a property of the inputs.
#pragma once

#include <stdint.h>

#include "pa_internal.cuh"

namespace pa {

// default limits of the product's waits
constexpr unsigned long long kWaitLimitNs = 4000000000ull;  // mbarrier phases: 4 s
constexpr unsigned long long kSpinLimitNs = 2000000000ull;  // shared-memory flags: 2 s
// longest single sleep of a thread waiting on an mbarrier before it checks the
// limit again
#ifndef PA_WAIT_SUSPEND_NS
#define PA_WAIT_SUSPEND_NS 20000
#endif
constexpr uint32_t kWaitSuspendNs = PA_WAIT_SUSPEND_NS;

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// The same, but a thread whose phase has not completed sleeps until it does,
// or for at most suspend_ns, instead of returning at once: waiting warps then
// take no issue slots from the warps that share their scheduler.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity,
                                                    uint32_t suspend_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(suspend_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with parity `parity` to complete.  Gives up
// (returns false) when another role of the CTA has given up, or after
// limit_ns, in which case it records the timeout and raises the abort flag.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* status,
                                         unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSuspendNs)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
  }
}

// Spin until ready() holds.  Gives up (returns false) when another role of the
// CTA has given up, or after limit_ns, in which case it records the timeout and
// raises the abort flag.
template <typename Ready>
__device__ __forceinline__ bool spin_until(Ready ready, volatile int* abort_flag, int* status,
                                           unsigned long long limit_ns = kSpinLimitNs) {
  if (ready()) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (ready()) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(status, kStatusWaitTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

}  // namespace pa
