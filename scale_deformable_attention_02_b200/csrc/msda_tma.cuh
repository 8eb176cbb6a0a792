// msda_tma.cuh -- tensor-copy (TMA) and mbarrier helpers of the tiled kernels
// (sm_100a, inline PTX).
//
// One thread of a CTA arms an mbarrier with the byte count it expects and
// issues the tensor copies; every thread then waits on the barrier's phase.
// Every wait is bounded: a phase that has not completed after kWaitTries
// tries (each try suspends the thread for up to about a microsecond) makes
// the wait return false instead of spinning for ever.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msda {

// Tries of one bounded wait: about a second at the suspend hint below.
constexpr int kWaitTries = 1 << 20;
constexpr uint32_t kWaitHintNs = 1000;

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
    // make the initialised barrier visible to the tensor-copy unit
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Retire the barrier before its shared memory is used for anything else.
__device__ __forceinline__ void mbar_inval(uint64_t *bar)
{
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Arrive on the barrier (the single expected arrival) and add `bytes` to the
// bytes the current phase waits for.
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{ .reg .pred q; mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2, %3; "
        "selp.u32 %0, 1, 0, q; }"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity), "r"(kWaitHintNs)
        : "memory");
    return done != 0;
}

// Wait until the barrier's phase with this parity has completed; false if it
// has not after kWaitTries tries.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    for (int i = 0; i < kWaitTries; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Order this thread's earlier shared-memory accesses (generic proxy) before
// later tensor copies into the same memory (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// One 5-d tiled tensor copy global -> shared memory of this CTA, completing
// on `bar`.  Coordinates outside the tensor read the fill value (zero); the
// innermost coordinate c0 stays 0 here, so it is always 16-byte aligned.
__device__ __forceinline__ void tma_load_5d(void *dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, int c4, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "r"(smem_addr(bar))
        : "memory");
}

}  // namespace msda
