// Bulk asynchronous copies from global into shared memory, completed on an
// mbarrier (PTX cp.async.bulk / mbarrier, sm_90 and later), and bounded waits.
// Copies are plain (never multicast); both addresses 16-byte aligned and the
// size a multiple of 16.
#pragma once

#include <stdint.h>

namespace moe {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

// Makes mbarrier initialisation visible to the asynchronous copy unit.
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// One arrival that also announces `bytes` of copies completing on this phase.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// One plain arrival (release semantics at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Named barrier `id` over `threads` threads (a multiple of 32) that also ORs a
// predicate across them: every participant gets the same answer.
__device__ __forceinline__ bool named_barrier_or(int id, int threads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(threads)
      : "memory");
  return r != 0;
}

// Tests the phase of the given parity; the thread may be suspended (up to
// about hint_ns) until it completes instead of returning at once.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_time_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Orders this thread's earlier generic-proxy accesses to shared memory before
// its later asynchronous-proxy ones (a buffer read by the CTA, then refilled).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// A wait gives up after about this long (timed with the global nanosecond
// timer, so the bound holds however long each suspended try lasts).
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr uint32_t kWaitHintNs = 20000;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity, kWaitHintNs)) return true;
  const uint64_t t0 = global_time_ns();
  while (!mbar_try_wait(bar, parity, kWaitHintNs))
    if (global_time_ns() - t0 > limit_ns) return false;
  return true;
}

// Waits of a staged kernel: the limit of its pipeline waits, and a test hook
// (off in every product call: withhold < 0) that makes the first CTA arm one
// unit's "full" barrier for 16 bytes without starting any copy for it, so
// that the waits on that unit run out while no copy is in flight for it. The
// waits that let started copies land before a CTA leaves always use
// kWaitLimitNs and skip the withheld unit.
struct WaitCfg {
  uint64_t limit_ns;
  int withhold;
};
constexpr WaitCfg kProductWaits = {kWaitLimitNs, -1};

}  // namespace moe
