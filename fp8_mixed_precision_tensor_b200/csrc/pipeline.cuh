// pipeline.cuh -- shared-memory barrier (mbarrier) helpers of the library's
// producer/consumer pipelines (the GEMMs' TMA rings).  Every wait is bounded by wall clock (%globaltimer):
// on timeout it raises FP8_STATUS_TIMEOUT and an abort flag of the CTA, so a
// pipeline that cannot make progress ends with a status instead of a hang.
#pragma once

#include "common.cuh"

namespace fp8lib {

constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s: far above any legitimate wait

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// One potentially blocking test of a barrier phase.  With the suspend-time
// hint the thread sleeps until the phase completes (or the hint elapses)
// instead of spinning, which keeps waiting warps off the issue slots and the
// memory-instruction queue that the TMA and tcgen05 instructions also use.
constexpr uint32_t kSuspendHintNs = 1000000;  // 1 ms per try; the caller bounds the total
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on one phase of an mbarrier.  Returns false on timeout (after
// raising the status bit and the CTA's abort flag) or when another role of
// the CTA has already aborted.  limit_ns: kTimeoutNs in the GEMMs.
__device__ __noinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                           uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_status, FP8_STATUS_TIMEOUT);
      *abort_flag = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
  return mbar_wait_for(bar, parity, abort_flag, kTimeoutNs);
}

// A wait used only while tearing down after an abort: bounded, no flag check.
__device__ __noinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kTimeoutNs) return;
  }
}


}  // namespace fp8lib
