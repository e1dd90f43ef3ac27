// Bounded waits on an mbarrier phase, shared by every kernel that waits and
// by tq_check_wait_expiry.  A wait polls the phase against a clock64 budget;
// on expiry it records TQ_ERR_TIMEOUT in the device error word (when `err`
// is not null) and returns false, so the caller can let its copies land,
// release what it holds and return instead of hanging.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

#include "tq_internal.h"

namespace tq {

// Default budget: about a second at the B200's clocks.
constexpr long long kWaitBudget = 1LL << 31;

// One test of the phase with the given parity: mbarrier.test_wait (a
// non-blocking poll) or, with TRY, mbarrier.try_wait (which may suspend the
// thread for a system-dependent time before reporting).
template <bool TRY>
__device__ __forceinline__ bool mbar_probe(uint32_t bar, uint32_t parity) {
  uint32_t done;
  if constexpr (TRY) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
  }
  return done != 0;
}

template <bool TRY>
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, unsigned* err,
                                             long long budget = kWaitBudget) {
  if (mbar_probe<TRY>(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_probe<TRY>(bar, parity)) {
    if (clock64() - t0 > budget) {
      if (err) atomicCAS(err, 0u, (unsigned)TQ_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

}  // namespace tq
