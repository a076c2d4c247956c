// Shared-memory pipelines fed by the bulk-copy engine: mbarrier helpers and
// 1-D bulk global->shared copies (cp.async.bulk, no multicast), used by the
// encoder and by the tensor-core decode kernel.  Every wait is bounded.
#pragma once

#include <stdint.h>

namespace q4kv {

constexpr unsigned kSpinLimit = 1u << 21;   // bounded mbarrier waits: ~2 s or more in all
constexpr unsigned kSuspendNs = 1000;       // hardware suspend hint of one try_wait

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}" ::"r"(smem_u32(bar))
               : "memory");
}
// An arrival by the threads where p holds, as one predicated instruction
// (no divergent branch around a single-lane arrival).
__device__ __forceinline__ void arrive_if(bool p, uint64_t* bar) {
  asm volatile("{\n .reg .pred q;\n .reg .b64 st;\n setp.ne.u32 q, %1, 0;\n @q mbarrier.arrive.shared::cta.b64 st, [%0];\n}"
               :: "r"(smem_u32(bar)), "r"(static_cast<uint32_t>(p)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// One try_wait: the thread is suspended (issuing nothing) until the phase
// completes or the hint runs out; true when the phase has completed.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(kSuspendNs)
      : "memory");
  return ok != 0;
}
// Bounded wait; false when the limit ran out.  The suspend hint is only an
// upper bound, so between tries the thread also sleeps, backing off from
// 32 ns to 1 us; the whole wait stays above two seconds before it gives up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned limit = kSpinLimit) {
  unsigned ns = 32;
  for (unsigned i = 0; i < limit; ++i) {
    if (mbar_try(bar, parity)) return true;
    __nanosleep(ns);
    ns = ns < 1024 ? 2 * ns : 1024;
  }
  return false;
}
// One test of the phase, never suspending the thread.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for a warp that has nothing else to do (a producer or a
// helper warp): test, then sleep ns0 doubling up to ns1 between tests, so its
// polling takes few issue slots from the warps sharing its scheduler.  A
// try_wait with a suspend hint polls far more often while it waits.  The
// limit (4 kSpinLimit tests, at least ~2 s when ns1 >= 64) is only a bound.
__device__ __forceinline__ bool mbar_wait_idle(uint64_t* bar, uint32_t parity, unsigned ns0, unsigned ns1) {
  unsigned ns = ns0;
  for (unsigned i = 0; i < 4 * kSpinLimit; ++i) {
    if (mbar_test(bar, parity)) return true;
    __nanosleep(ns);
    ns = ns < ns1 ? 2 * ns : ns1;
  }
  return false;
}
// bytes and both addresses must be multiples of 16
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

}  // namespace q4kv
