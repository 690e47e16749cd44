// bnbq_async.cuh -- bulk asynchronous copies into shared memory for the staged kernels (sm_100a).
//
// A tile of global memory is copied into shared memory by one cp.async.bulk (the copy engine of
// sm_90 and later; no tensor map, no multicast), which signals an mbarrier with the bytes it
// delivered; the consuming threads wait on the barrier's phase.  Every wait is bounded by a clock
// budget and reports a timeout instead of spinning on; a kernel that sees one sets kFlagTimeout.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace bnbq {

constexpr unsigned kFlagTimeout = 0x4u;  // mirrors BNBQ_FLAG_TIMEOUT in include/bnbq.h

constexpr long long kWaitCycles = 1ll << 31;  // about a second at the B200's clocks

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Makes initialised barriers visible to the copy engine (before the first copy that signals them).
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Orders this thread's earlier shared-memory accesses before later bulk copies into shared memory.
__device__ __forceinline__ void async_proxy_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// One arrival that also announces `bytes` of copies for the barrier's current phase.
__device__ __forceinline__ void mbar_arrive_expect(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

// Copy `bytes` (a multiple of 16; both addresses 16-byte aligned) from global to shared memory,
// completing `bytes` of the barrier's transaction count.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return done != 0;
}

// Hint: bring `bytes` (a multiple of 16; address 16-byte aligned) of global memory into L2.
__device__ __forceinline__ void l2_prefetch(const void* src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Wait for the phase of parity `parity` to complete; false if it has not within kWaitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity))
        if (clock64() - t0 > kWaitCycles) return false;
    return true;
}

}  // namespace bnbq
