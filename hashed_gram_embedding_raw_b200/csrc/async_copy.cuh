// async_copy.cuh -- bulk (TMA) copies into shared memory and the mbarriers
// that track them, shared by the PLE kernels. Every wait is bounded in time:
// a wait that runs out returns false, and the caller raises
// ENGRAM_DEVERR_COPY_TIMEOUT and ends promptly instead of hanging.
#pragma once

#include "common.cuh"

namespace engram {
namespace ple {

constexpr uint64_t kCopyWaitNs = 500ull * 1000 * 1000;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// One contiguous global -> shared copy by the bulk-copy (TMA) engine,
// completing `bytes` of transaction count on `bar`. Both addresses 16-byte
// aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Waits (bounded by limit_ns) for phase `parity` of `bar`; false on timeout.
// The clock is read once every 64 polls, so a poll costs little issue time.
// limit_ns == 0 tests the phase once without waiting (a test hook's bound).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = kCopyWaitNs)
{
    const uint32_t addr = smem_u32(bar);
    if (limit_ns == 0) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(addr), "r"(parity)
                     : "memory");
        return done != 0;
    }
    uint64_t t0 = 0;
    for (uint32_t spin = 0;; ++spin) {
        uint32_t done;
        asm volatile("{\n\t.reg .pred p;\n\t"
                     "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(done)
                     : "r"(addr), "r"(parity)
                     : "memory");
        if (done)
            return true;
        if ((spin & 63) == 0) {
            uint64_t now;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
            if (spin == 0)
                t0 = now;
            else if (now - t0 > limit_ns)
                return false;
        }
    }
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Arrival with release semantics: this thread's earlier shared-memory
// accesses are visible to a thread that then sees the phase complete.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

} // namespace ple
} // namespace engram
