// mbar.cuh -- bulk asynchronous copies (cp.async.bulk, the TMA engine's
// untiled form) and mbarriers with bounded waits, shared by the kernels that
// stage rows in shared memory or wait on tensor-core completions.
//
// Every wait is bounded in global time: a wait that runs out returns false,
// and the caller records it in its translation unit's sticky timeout flag
// (read by hyena_device_timeouts) instead of spinning on.
#pragma once

#include <stdint.h>

namespace hyena {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
// make initialised mbarriers visible to the async proxy (before the barrier
// that publishes them to the other threads)
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// this thread's arrival, expecting `bytes` of asynchronous copies
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// Bulk copy of `bytes` (a multiple of 16; both addresses 16-byte aligned)
// from global to this CTA's shared memory; completion counts on `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// L2 cache policy under which the lines a copy fills are the first to be
// evicted: for data read once (filter spectrum rows), so that it does not
// push out data that is read again (a wave's four-step scratch).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// bulk_g2s under an L2 cache policy
__device__ __forceinline__ void bulk_g2s_policy(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                                uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(pol)
      : "memory");
}

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, multiple of 16 bytes).
__device__ __forceinline__ void bulk_prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase `phase` of an mbarrier to complete, bounded in time:
// each try suspends for at most kMbarSuspendNs, and the wait gives up once
// limit_ns of global time have passed since it started (returns false).
constexpr unsigned kMbarSuspendNs = 20000;                   // 20 us per try
constexpr unsigned long long kMbarWaitLimitNs = 200000000ull; // 0.2 s per wait
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase,
                                          unsigned long long limit_ns = kMbarWaitLimitNs) {
  const unsigned long long t0 = globaltimer_ns();
  for (;;) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred P1;\n\tmbarrier.try_wait.parity.shared::cta.b64 P1, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, P1;\n\t}\n"
        : "=r"(done)
        : "r"(bar), "r"(phase), "r"(kMbarSuspendNs)
        : "memory");
    if (done) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

}  // namespace hyena
