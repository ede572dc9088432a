// tma.cuh -- mbarrier and bulk-copy (TMA, non-tensor) helpers, inline PTX for sm_100a.
//
// Every wait is bounded: after kSpinLimit failed polls (each a suspended wait
// of up to kSuspendNs, or a short sleep) the waiter records an
// error code in the handle's device error word and carries on, so a broken
// pipeline ends the kernel with a reported error instead of a hang.  All
// addresses a kernel computes come from item metadata, never from loaded
// data, so proceeding after a timeout stays in bounds.
#pragma once

#include <stdint.h>

namespace moe {

constexpr uint32_t kSpinLimit = 1u << 20;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// The waiting thread is suspended in hardware until the phase completes or
// kSuspendNs pass, so a waiting warp does not spin on the issue slots that the
// working warps of its scheduler need (measured: 20, 100 or 1000 ns, or no
// suspension at all, give the same times).
constexpr uint32_t kSuspendNs = 1000;

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Non-blocking test of the same condition.
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
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

// Wait for the phase with the given parity to complete; bounded.  Once any
// agent of the kernel has reported an error the wait gives up early, so a
// broken pipeline unwinds in one timeout rather than one per remaining wait.
// The first (suspended) test is inline; the bounded loop is out of line, so
// the many call sites stay small in the instruction cache.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t *bar, uint32_t parity, int *err, int code)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 1023u && *reinterpret_cast<volatile int *>(err) != 0) return false;
    }
    atomicCAS(err, 0, code);
    return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *err, int code)
{
    return mbar_try_wait(bar, parity) || mbar_wait_slow(bar, parity, err, code);
}

// A bounded wait that does not give up early on another agent's error: used
// only to drain copies before the CTA exits.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return;
}

// Contiguous global -> shared copy completed on `bar` (bytes % 16 == 0, both
// addresses 16-byte aligned).  A CTA is its own cluster of one here.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// The same with an L2 eviction-priority hint (weights stream once).
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Barriers among a subset of the CTA's warps (named barriers 1 and 2); the
// other warps never join them.
__device__ __forceinline__ void consumer_sync(int n_threads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(n_threads) : "memory");
}

__device__ __forceinline__ void group_sync(int id, int n_threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n_threads) : "memory");
}

}  // namespace moe
