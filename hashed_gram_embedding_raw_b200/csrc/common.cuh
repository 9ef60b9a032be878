// common.cuh -- helpers shared by the Engram kernels (sm_100a).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "engram.h"

namespace engram {

constexpr unsigned kFull = 0xffffffffu;

// Per-device error word (ENGRAM_DEVERR_* bits); zero when the module loads.
// Kernels OR bits into it instead of trapping.
__device__ unsigned int g_device_error;

__device__ __forceinline__ void raise_device_error(unsigned bits)
{
    atomicOr(&g_device_error, bits);
}

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ------------------------------------------------------------- modular math

__host__ __device__ __forceinline__ uint64_t mulhi64(uint64_t a, uint64_t b)
{
#ifdef __CUDA_ARCH__
    return __umul64hi(a, b);
#else
    return (uint64_t)(((unsigned __int128)a * b) >> 64);
#endif
}

// Barrett reduction: n mod p for any 64-bit n and 1 <= p < 2^63, where
// magic = floor((2^64 - 1) / p) >= 2^64 / p - 1. The estimate
// q = floor(n * magic / 2^64) then satisfies n/p - 1 < n*magic/2^64 <= n/p,
// so q is floor(n/p) or one less and r = n - q*p lies in [0, 2p): a single
// conditional subtraction completes the remainder.
__host__ __device__ __forceinline__ uint64_t barrett_mod(uint64_t n, uint64_t p, uint64_t magic)
{
    const uint64_t q = mulhi64(n, magic);
    const uint64_t r = n - q * p;
    return r >= p ? r - p : r;
}

// Remainder of a signed a by p > 0 in [0, p) ("positive remainder").
// For a < 0 write a = -(u + 1) with u = ~a >= 0; then a mod p = p - 1 - (u mod p).
__host__ __device__ __forceinline__ int64_t floor_mod(int64_t a, uint64_t p, uint64_t magic)
{
    const bool neg = a < 0;
    const uint64_t u = neg ? ~(uint64_t)a : (uint64_t)a;
    const uint64_t r = barrett_mod(u, p, magic);
    return (int64_t)(neg ? p - 1 - r : r);
}

// --------------------------------------------------------- memory helpers

// 16-byte read-only load that does not allocate in L1 (table rows and
// gradients are touched once per launch).
__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p));
    return v;
}

// 16-byte streaming store (evict-first): outputs are written once.
__device__ __forceinline__ void st_stream(uint4 *p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_stream(float4 *p, float4 v)
{
    asm volatile("st.global.cs.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

// Load with acquire semantics at device scope (pairs with a releasing write).
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned *p)
{
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t lanemask_lt()
{
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Exclusive scan of one value per thread over the block (blockDim.x a
// multiple of 32, at most 1024). s_warp holds 32 words of shared scratch.
// Every thread gets the block total in *total when total != nullptr. TRAIL =
// false leaves out the closing barrier that protects s_warp from the next
// scan; the caller must then pass a block barrier before reusing s_warp.
template <bool TRAIL = true>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *s_warp,
                                                         uint32_t *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(kFull, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        s_warp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        uint32_t s = lane < nw ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(kFull, s, o);
            if (lane >= o)
                s += y;
        }
        if (lane < nw)
            s_warp[lane] = s;
    }
    __syncthreads();
    const uint32_t before = wid ? s_warp[wid - 1] : 0u;
    if (total)
        *total = s_warp[nw - 1];
    if constexpr (TRAIL)
        __syncthreads();
    return before + x - v;
}

// The same scan over 64-bit values (no total); s_warp holds 32 words.
template <bool TRAIL = true>
__device__ __forceinline__ unsigned long long block_exclusive_scan64(unsigned long long v,
                                                                    unsigned long long *s_warp)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    unsigned long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(kFull, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        s_warp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        unsigned long long s = lane < nw ? s_warp[lane] : 0ull;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(kFull, s, o);
            if (lane >= o)
                s += y;
        }
        if (lane < nw)
            s_warp[lane] = s;
    }
    __syncthreads();
    const unsigned long long before = wid ? s_warp[wid - 1] : 0ull;
    if constexpr (TRAIL)
        __syncthreads();
    return before + x - v;
}

// -------------------------------------------------------- sequence bounds

// Largest s < nseq with cu[s] <= t (cu[0] = 0 <= t for well-formed bounds).
__device__ __forceinline__ int32_t find_sequence(const int32_t *__restrict__ cu, int32_t nseq,
                                                 int64_t t)
{
    int32_t lo = 0, hi = nseq - 1;
    while (lo < hi) {
        const int32_t mid = (lo + hi + 1) >> 1;
        if (__ldg(cu + mid) <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// find_sequence for a t shared by the whole warp: each round the 32 lanes probe
// 32 evenly spaced bounds at once, so nseq <= 32 takes one round of loads
// and 1,024 two, instead of a chain of log2(nseq) dependent loads.
__device__ __forceinline__ int32_t find_sequence_warp(const int32_t *__restrict__ cu,
                                                      int32_t nseq, int64_t t)
{
    const int lane = threadIdx.x & 31;
    int32_t lo = 0, hi = nseq - 1; // the answer lies in [lo, hi]; cu[lo] <= t
    while (lo < hi) {
        const int32_t step = (hi - lo + 32) / 32; // ceil((hi - lo + 1) / 32)
        const int32_t p = lo + lane * step;
        const bool le = p <= hi && (p == lo || __ldg(cu + p) <= t);
        const uint32_t m = __ballot_sync(kFull, le);
        const int32_t k = 31 - __clz(m); // lane 0 always qualifies
        lo = lo + k * step;
        hi = min(hi, lo + step - 1);
    }
    return lo;
}

// Flags malformed cu_seqlens (not 0 .. T, or decreasing). Grid-strided.
__device__ __forceinline__ void check_cu_seqlens(const int32_t *__restrict__ cu, int32_t nseq,
                                                 int64_t T)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i <= nseq; i += stride) {
        const int64_t c = __ldg(cu + i);
        const bool bad = (i == 0 && c != 0) || (i == nseq && c != T) ||
                         (i < nseq && c > __ldg(cu + i + 1));
        if (bad)
            raise_device_error(ENGRAM_DEVERR_CU_SEQLENS);
    }
}

} // namespace engram
