// pipeline.cuh -- bulk-copy (TMA) and mbarrier primitives for the persistent
// producer/consumer kernels (sm_100a, inline PTX).
//
// Every wait is bounded in wall-clock time: after kWaitLimitNs without the
// awaited phase completing, the waiter gives up and the caller reports
// RSSM_ERR_TIMEOUT in the status word instead of spinning forever.  Bulk
// copies are plain (no cluster multicast) and only ever read this GPU's own
// memory.
#pragma once
#include <stdint.h>

namespace rssm {

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of the given parity to complete.  Returns false when
// `limit_ns` of wall-clock time pass first, or -- if `abort` is given -- as
// soon as another warp of the CTA has set *abort (its peer stopped, so the
// awaited arrival may never come).  Waits for this thread's own bulk copies
// in flight pass no abort flag: those copies complete on their own.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs,
                                          volatile int *abort = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (global_ns() - t0 > limit_ns) return false;
      if (abort && *abort) return false;
    }
  }
}

// Record bulk copies armed by a stager warp: per record buffer, whether it
// has been armed and the phase parity of its latest arming.  On exit the
// stager waits (bounded, regardless of any abort) for the latest phase of
// every armed buffer, so that no record copy is in flight when the CTA ends.
struct ArmedRecords {
  uint32_t armed = 0, parity = 0;
  __device__ __forceinline__ void arm(int rb, uint32_t ph) {
    armed |= 1u << rb;
    parity = (parity & ~(1u << rb)) | (ph << rb);
  }
  __device__ __forceinline__ void drain(uint64_t *rfull, int nr) const {
    for (int r = 0; r < nr; ++r)
      if (armed & (1u << r)) mbar_wait(&rfull[r], (parity >> r) & 1u);
  }
};

// Global -> shared bulk copy completing on `bar` (bytes % 16 == 0, both
// addresses 16-byte aligned).
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// Order this thread's generic-proxy shared-memory accesses before later
// async-proxy (bulk copy) writes to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Named barrier over `n` threads (the consumer warps), id != 0.
__device__ __forceinline__ void bar_sync(uint32_t id, uint32_t n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Named barrier that also ORs a predicate across the participating threads.
__device__ __forceinline__ bool bar_or(uint32_t id, uint32_t n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.or.pred q, %2, %3, p;\n"
      " selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

}  // namespace rssm
