// tma.cuh -- bulk-copy (TMA engine) and mbarrier helpers for sm_100a.
//
// Only non-multicast copies from this GPU's own global memory into the
// issuing CTA's shared memory are used.  Every wait on an mbarrier is
// bounded by the global timer; a wait that gives up returns false and the
// caller latches MOE_FP4_ETIMEOUT instead of spinning forever.
#pragma once
#include <cstdint>

namespace moe {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make initialised barriers visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// L2 policy for data read exactly once (expert weights): evict first.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Global -> shared bulk copy (no multicast); completes `bytes` on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Same without an L2 eviction hint (small operands that other CTAs read too).
__device__ __forceinline__ void bulk_g2s_nohint(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// One bounded probe of phase `parity`: the hardware may suspend the thread
// for up to `hint_ns` (at most ~0.5 ms) waiting for the phase instead of a
// hot spin.
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity, uint32_t hint_ns = 500000u) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Non-blocking probe: has phase `parity` of `bar` completed?
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Raise the transaction count of the current phase by `bytes` without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Wait for phase `parity` of `bar` by polling (non-blocking probes with a
// short sleep between them): the phase is seen within tens of nanoseconds
// whichever agent completes it.  Same bounds and abort rules as mbar_wait.
__device__ __forceinline__ bool mbar_poll(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns = 1000000000ull) {
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        __nanosleep(32);
        if (mbar_test(bar, parity)) return true;
        if ((n & 15) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort = 1;
                return false;
            }
        }
    }
}

// Wait for phase `parity` of `bar` to complete.  Returns false at once when
// *abort is set, and sets it (false) after ~timeout_ns: the first wait of a
// CTA that gives up makes every later wait of that CTA return immediately, so
// a broken pipeline costs one timeout, not one per item.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns = 1000000000ull) {
    const uint32_t hint = timeout_ns < 500000ull ? static_cast<uint32_t>(timeout_ns) : 500000u;
    if (mbar_try_wait(bar, parity, hint)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity, hint)) {
        if (*abort) return false;
        if (global_timer_ns() - t0 > timeout_ns) {
            *abort = 1;
            return false;
        }
    }
    return true;
}

}  // namespace moe
