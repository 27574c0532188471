// Shared-memory pipeline primitives for the sm_100a kernels: mbarriers with bounded waits.
//
// Every wait of one thread on another gives up after a time limit (%globaltimer): it sets a
// bit in the library's sticky device error word and a CTA-wide abort flag, so a stuck pipeline
// ends with an error the host can read instead of a hung GPU.
#pragma once

#include <cstdint>

namespace fi {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

// One bounded, suspending test of the phase: the thread sleeps in hardware until the phase
// completes or kWaitSliceNs pass.
constexpr uint32_t kWaitSliceNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity), "r"(kWaitSliceNs)
      : "memory");
  return done != 0;
}

// Wait for phase `parity` of `bar` to complete. Returns false (raising the CTA's abort flag and
// err_bit in *err_word) if it has not after timeout_ns, or at once if the CTA has aborted.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint64_t timeout_ns, unsigned* err_word, unsigned err_bit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      *abort_flag = 1;
      atomicOr(err_word, err_bit);
      return false;
    }
  }
}

}  // namespace fi
