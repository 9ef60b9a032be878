// ple_conv.cuh -- the PLE layer's branch-local RMS norm and causal short
// convolution (engram page, Qwen3_8_FlashNextPLELayer: norm_conv, conv1d,
// _causal_short_conv; layers page, Qwen3_8_FlashNextGroupedRMSNorm).
//
// x is [T, C] with C = groups * G: a token row holds `groups` HyperConnection
// branches of G features each. For every branch slice of every token,
//   n     = x * rsqrt(mean over the slice of x^2 + eps)        (optional norm)
//   y[c]  = bias[c] + sum over k < K with t - k*d >= sequence start of
//           w'[c][k] * n[t - k*d][c],   w'[c][k] = conv_w[c][K-1-k] * (1 + norm_w[c])
//   out   = x + y * sigmoid(y)                        (SiLU and residual optional)
//
// One block per (branch, token range); the ranges of a branch are cut evenly
// among sms / groups blocks, so one wave fills the GPU. A block walks its
// range in chunks of kChunk rows, with one __syncthreads per chunk:
//   - thread 0 keeps the rows of the next two chunks on their way into L2
//     with bulk prefetches (cp.async.bulk.prefetch.L2, fire and forget);
//   - pass 1, one warp per row: the warp sums the squares of the row's branch
//     slice (16-byte loads, several in flight per lane) and one lane stores
//     the row's inverse RMS in shared memory; threads also note each row's
//     count of in-sequence history taps;
//   - pass 2, channel-parallel: thread v owns 4 (for branches wider than
//     2,560: 8) channels and walks the chunk's rows four at a time, reading
//     its channels again (L2 hits) with the next four rows' loads in flight.
//     It keeps the normalised values of its own channels for the last
//     halo + kRows rows in a private part of shared memory (no other thread
//     reads them, so they need no barrier) and forms the convolution, SiLU and
//     residual with packed f32x2 arithmetic; outputs leave with streaming
//     stores.
// The halo rows before a block's range are read and normalised but produce no
// output (0.5 % extra reads on the page's shape).
#pragma once

#include <cuda_bf16.h>
#include <type_traits>

#include "common.cuh"

namespace engram {
namespace ple {

constexpr int kRows = 4;                 // rows per pass-2 step
constexpr int kChunk = 40;               // rows per chunk (one barrier each)
constexpr int kMaxTaps = 8;              // largest kernel width
constexpr int kNarrowThreads = 640;      // 4 channels per thread up to G = 2560
constexpr int kWideThreads = 512;        // 8 channels per thread up to G = 4096
constexpr int kHeaderBytes = 2 * kChunk * 8;  // inverse RMS and tap counts of two chunks
constexpr size_t kSmemLimit = 227 * 1024;

struct ConvArgs {
    const void *x;
    void *out;
    const int32_t *cu;
    int32_t nseq;
    int64_t T;
    int32_t C, G;
    int32_t bpg;        // blocks per branch
    int32_t nth;        // active threads per block = G / channels per thread
    const void *norm_w, *conv_w, *bias;
    int32_t wdtype;
    float eps, inv_G;
    int32_t K, dil, halo;
    int32_t norm_slots; // rows of the private normalised history (halo + kRows)
    uint32_t flags;     // ENGRAM_CONV_* bits
    int32_t reg_bufs;   // residue-class kernel: row buffers (of 8 rows each)
    int32_t pitch;      // residue-class kernel: bytes per buffered row
    int32_t classes;    // residue-class kernel: residues with rows, min(dil, T)
    uint64_t cross_wait_ns; // residue-class kernel: bound of a wait on other warps
    float *inv_out;         // [T][C / G] inverse RMS of every branch slice, or null
    int32_t groups;         // C / G
};

// Shared memory: inverse RMS [2][kChunk] float and history-tap counts
// [2][kChunk] int32 (kHeaderBytes), then the private rings
// [norm_slots][chan / 4][nth] float4.
__host__ __device__ constexpr size_t smem_bytes(int norm_slots, int nth, int chan)
{
    return (size_t)kHeaderBytes + (size_t)norm_slots * nth * chan * sizeof(float);
}

// Starts moving `bytes` (a multiple of 16, 16-byte aligned) from global
// memory into L2; nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// B bytes (8 or 16) of read-only global data into B / 4 words.
template <int B>
__device__ __forceinline__ void load_global(const void *p, uint32_t *w)
{
    if constexpr (B == 8) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];"
                     : "=r"(w[0]), "=r"(w[1])
                     : "l"(p));
    } else {
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "l"(p));
    }
}

// ------------------------------------------------------ element conversion

// N consecutive elements of T packed in N * sizeof(T) / 4 32-bit words.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    template <int N>
    __device__ static void unpack(const uint32_t *w, float *f)
    {
#pragma unroll
        for (int i = 0; i < N; ++i)
            f[i] = __uint_as_float(w[i]);
    }
    template <int N>
    __device__ static void pack(const float *f, uint32_t *w)
    {
#pragma unroll
        for (int i = 0; i < N; ++i)
            w[i] = __float_as_uint(f[i]);
    }
};

template <>
struct Elem<__nv_bfloat16> {
    // a bf16 value is the upper half of the fp32 with the same bits
    template <int N>
    __device__ static void unpack(const uint32_t *w, float *f)
    {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    // round to nearest even, element 2i in the low half
    template <int N>
    __device__ static void pack(const float *f, uint32_t *w)
    {
#pragma unroll
        for (int i = 0; i < N / 2; ++i)
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[i]) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
    }
};

template <>
struct Elem<__half> {
    template <int N>
    __device__ static void unpack(const uint32_t *w, float *f)
    {
#pragma unroll
        for (int i = 0; i < N / 2; ++i)
            asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                "cvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
                : "=f"(f[2 * i]), "=f"(f[2 * i + 1])
                : "r"(w[i]));
    }
    template <int N>
    __device__ static void pack(const float *f, uint32_t *w)
    {
#pragma unroll
        for (int i = 0; i < N / 2; ++i)
            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w[i]) : "f"(f[2 * i + 1]), "f"(f[2 * i]));
    }
};

// B bytes (8, 16 or 32) to global memory with streaming stores.
template <int B>
__device__ __forceinline__ void store_words(void *p, const uint32_t *w)
{
    if constexpr (B == 8) {
        asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(w[0]), "r"(w[1])
                     : "memory");
    } else {
#pragma unroll
        for (int q = 0; q < B / 16; ++q)
            st_stream(reinterpret_cast<uint4 *>(p) + q,
                      make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
    }
}

__device__ __forceinline__ float load_weight(const void *w, int32_t dtype, int64_t i)
{
    if (dtype == ENGRAM_F32)
        return __ldg(static_cast<const float *>(w) + i);
    const unsigned short b = __ldg(static_cast<const unsigned short *>(w) + i);
    if (dtype == ENGRAM_BF16)
        return __uint_as_float((uint32_t)b << 16);
    return __half2float(__ushort_as_half(b));
}

// ------------------------------------------------------------- arithmetic

// 2^x and 1/x on the special-function unit (flush-to-zero forms).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// y * sigmoid(y) = y / (1 + e^-y), with e^-y = 2^(-y log2 e), for a pair.
__device__ __forceinline__ float2 silu2(float2 y)
{
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 z = __fmul2_rn(y, make_float2(kNegLog2e, kNegLog2e));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(z.x), ex2_approx(z.y)),
                                make_float2(1.f, 1.f));
    return __fmul2_rn(y, make_float2(rcp_approx(d.x), rcp_approx(d.y)));
}

// Sums four per-lane values over the warp in 6 shuffles (each exchange step
// hands half of the values still held to the partner): lane l ends with the
// total of value 2 * bit4(l) + bit3(l), so lanes 0, 8, 16, 24 hold 0, 1, 2, 3.
__device__ __forceinline__ float warp_sum4(float v0, float v1, float v2, float v3, int lane)
{
    const bool h16 = lane & 16;
    float a0 = h16 ? v2 : v0, a1 = h16 ? v3 : v1;
    const float s0 = h16 ? v0 : v2, s1 = h16 ? v1 : v3;
    a0 += __shfl_xor_sync(kFull, s0, 16);
    a1 += __shfl_xor_sync(kFull, s1, 16);
    const bool h8 = lane & 8;
    float b = h8 ? a1 : a0;
    b += __shfl_xor_sync(kFull, h8 ? a0 : a1, 8);
    b += __shfl_xor_sync(kFull, b, 4);
    b += __shfl_xor_sync(kFull, b, 2);
    b += __shfl_xor_sync(kFull, b, 1);
    return b;
}

// ------------------------------------------------------------------ kernel

// XT: element type of x; OT: of out; KT: kernel width (0 = runtime, <= 8);
// CH: channels per thread in pass 2 (4 or 8); SAVE: also store every output
// row's inverse RMS to inv_out.
template <typename XT, typename OT, int KT, int CH, bool SAVE>
__global__ void __launch_bounds__(CH == 4 ? kNarrowThreads : kWideThreads, 1)
    short_conv_kernel(const ConvArgs a)
{
    constexpr int XB = CH * (int)sizeof(XT);  // input bytes per thread and row
    constexpr int VB = XB < 16 ? XB : 16;     // bytes per load
    constexpr int NV = XB / VB;               // loads per thread and row (1 or 2)
    constexpr int NW = VB / 4;                // words per load
    constexpr int EV = VB / (int)sizeof(XT);  // channels per load
    constexpr int OB = EV * (int)sizeof(OT);  // output bytes per load's channels
    constexpr int NP = CH / 2;                // channel pairs
    constexpr int NQ = CH / 4;                // float4 groups of the private ring
    constexpr int KM = KT ? KT : kMaxTaps;
    constexpr int RV = 16 / (int)sizeof(XT);  // elements per 16-byte load in pass 1
    constexpr int P1 = 10;                    // pass-1 loads per lane in flight
    extern __shared__ __align__(128) unsigned char smem[];

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    const bool active = tid < a.nth;
    const int K = KT ? KT : a.K;
    const int m = blockIdx.x / a.bpg, j = blockIdx.x - m * a.bpg;
    const int64_t ta = a.T * j / a.bpg, tb = a.T * (j + 1) / a.bpg;
    if (ta >= tb)
        return;
    const int64_t tlo = ta - a.halo > 0 ? ta - a.halo : 0;

    float *inv_s = reinterpret_cast<float *>(smem);                      // [2][kChunk]
    int32_t *nv_s = reinterpret_cast<int32_t *>(smem + 2 * kChunk * 4);  // [2][kChunk]
    float4 *nring = reinterpret_cast<float4 *>(smem + kHeaderBytes);

    // weights of this thread's channels, in pairs; tap k looks k * dil rows
    // back and carries the norm's (1 + w) scale
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    float2 wk[KM][NP];
    float2 bias[NP];
#pragma unroll
    for (int e = 0; e < CH; ++e) {
        const int64_t c = (int64_t)m * a.G + (int64_t)(tid + (e / EV) * a.nth) * EV + e % EV;
        const float scale =
            active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
        const float b = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
        if (e & 1)
            bias[e / 2].y = b;
        else
            bias[e / 2].x = b;
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            float w = 0.f;
            if (active && k < K)
                w = (a.conv_w ? load_weight(a.conv_w, a.wdtype, c * K + (K - 1 - k)) : 1.f) *
                    scale;
            if (e & 1)
                wk[k][e / 2].y = w;
            else
                wk[k][e / 2].x = w;
        }
    }

    const uint32_t row_bytes = (uint32_t)a.G * sizeof(XT);
    const int nvec = (int)(row_bytes / 16);  // 16-byte vectors per branch slice
    const char *xbranch = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    const char *xmine = xbranch + (size_t)tid * VB;
    const int64_t xrow = (int64_t)a.C * sizeof(XT);
    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;
    char *out = static_cast<char *>(a.out);

    // thread 0: rows of the first two chunks towards L2
    int64_t pf = tlo;
    if (tid == 0)
        for (const int64_t end = min64(tb, tlo + 2 * kChunk); pf < end; ++pf)
            prefetch_l2(xbranch + pf * xrow, row_bytes);

    int nslot = 0;  // private-ring slot of the next pass-2 row
    for (int64_t c0 = tlo, chunk = 0; c0 < tb; c0 += kChunk, ++chunk) {
        const int rc = (int)min64(kChunk, tb - c0);
        const int buf = (int)(chunk & 1);
        if (tid == 0)
            for (const int64_t end = min64(tb, c0 + 3 * kChunk); pf < end; ++pf)
                prefetch_l2(xbranch + pf * xrow, row_bytes);

        // ---- pass 1: inverse RMS of every row, one warp per row
        for (int r = wid; r < rc; r += nw) {
            const char *row = xbranch + (c0 + r) * xrow;
            float2 ss = make_float2(0.f, 0.f);
            for (int v0 = 0; v0 < nvec; v0 += 32 * P1) {
                uint32_t w[P1][4];
#pragma unroll
                for (int u = 0; u < P1; ++u) {
                    const int v = v0 + u * 32 + lane;
                    if (v < nvec)
                        load_global<16>(row + (size_t)v * 16, w[u]);
                    else
                        w[u][0] = w[u][1] = w[u][2] = w[u][3] = 0u;
                }
#pragma unroll
                for (int u = 0; u < P1; ++u) {
                    float f[RV];
                    Elem<XT>::template unpack<RV>(w[u], f);
#pragma unroll
                    for (int e = 0; e < RV; e += 2) {
                        const float2 x2 = make_float2(f[e], f[e + 1]);
                        ss = __ffma2_rn(x2, x2, ss);
                    }
                }
            }
            float tot = ss.x + ss.y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                tot += __shfl_xor_sync(kFull, tot, o);
            if (lane == 0) {
                const float iv = do_norm ? rsqrtf(fmaf(tot, a.inv_G, a.eps)) : 1.f;
                inv_s[buf * kChunk + r] = iv;
                if (SAVE && c0 + r >= ta)  // (halo rows belong to the block before)
                    a.inv_out[(c0 + r) * a.groups + m] = iv;
            }
        }
        // in-sequence history taps of every row of the chunk
        for (int r = tid; r < rc; r += blockDim.x) {
            const int64_t t = c0 + r;
            const int64_t start =
                a.cu != nullptr ? (int64_t)__ldg(a.cu + find_sequence(a.cu, a.nseq, t)) : 0;
            const int64_t back = t - start;
            nv_s[buf * kChunk + r] = back >= a.halo ? K - 1
                                     : back <= 0    ? 0
                                                    : min(K - 1, (int)back / a.dil);
        }
        __syncthreads();

        // ---- pass 2: normalise, convolve, SiLU, residual, four rows at a time
        if (active) {
            uint32_t xn[kRows][NV][NW];
            auto load_rows = [&](int g) {
#pragma unroll
                for (int i = 0; i < kRows; ++i)
#pragma unroll
                    for (int q = 0; q < NV; ++q) {
                        if (g + i < rc)
                            load_global<VB>(xmine + (c0 + g + i) * xrow + (size_t)q * a.nth * VB,
                                            xn[i][q]);
                        else
#pragma unroll
                            for (int w = 0; w < NW; ++w)
                                xn[i][q][w] = 0u;
                    }
            };
            load_rows(0);
            for (int g = 0; g < rc; g += kRows) {
                const int nb = min(kRows, rc - g);
                float xv[kRows][CH];
#pragma unroll
                for (int i = 0; i < kRows; ++i)
#pragma unroll
                    for (int q = 0; q < NV; ++q)
                        Elem<XT>::template unpack<EV>(xn[i][q], &xv[i][q * EV]);
                load_rows(g + kRows);

                int nvr[kRows];
                float inv[kRows];
#pragma unroll
                for (int i = 0; i < kRows; ++i) {
                    nvr[i] = i < nb ? nv_s[buf * kChunk + g + i] : 0;
                    inv[i] = i < nb ? inv_s[buf * kChunk + g + i] : 0.f;
                }
                const int64_t tg = c0 + g;
                const bool fast = nb == kRows && tg >= ta && nvr[0] == K - 1 &&
                                  nvr[1] == K - 1 && nvr[2] == K - 1 && nvr[3] == K - 1;

                // normalise into the private ring; the current-row tap starts y
                float2 y[kRows][NP];
#pragma unroll
                for (int i = 0; i < kRows; ++i) {
                    const float2 inv2 = make_float2(inv[i], inv[i]);
                    float2 n[NP];
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        n[p] = __fmul2_rn(make_float2(xv[i][2 * p], xv[i][2 * p + 1]), inv2);
                        y[i][p] = __ffma2_rn(wk[0][p], n[p], bias[p]);
                    }
                    if (KM > 1 && (fast || i < nb)) {
                        int ns = nslot + i;
                        if (ns >= a.norm_slots)
                            ns -= a.norm_slots;
                        float4 *dst = nring + ns * NQ * a.nth + tid;
#pragma unroll
                        for (int q = 0; q < NQ; ++q)
                            dst[q * a.nth] = make_float4(n[2 * q].x, n[2 * q].y, n[2 * q + 1].x,
                                                         n[2 * q + 1].y);
                    }
                }

                // earlier rows' taps from the private ring
#pragma unroll
                for (int k = 1; k < KM; ++k) {
                    if (k >= K)
                        break;
#pragma unroll
                    for (int i = 0; i < kRows; ++i) {
                        if (!fast && (i >= nb || k > nvr[i]))
                            continue;
                        // slot of row i - k * dil of the group: i - k * dil
                        // lies in [-halo, kRows - 1], one correction either way
                        int hs = nslot + i - k * a.dil;
                        if (hs < 0)
                            hs += a.norm_slots;
                        else if (hs >= a.norm_slots)
                            hs -= a.norm_slots;
                        const float4 *h = nring + hs * NQ * a.nth + tid;
#pragma unroll
                        for (int q = 0; q < NQ; ++q) {
                            const float4 v = h[q * a.nth];
                            y[i][2 * q] =
                                __ffma2_rn(wk[k][2 * q], make_float2(v.x, v.y), y[i][2 * q]);
                            y[i][2 * q + 1] = __ffma2_rn(wk[k][2 * q + 1], make_float2(v.z, v.w),
                                                         y[i][2 * q + 1]);
                        }
                    }
                }

                // SiLU and residual over all rows at once, then the stores
                if (do_silu) {
#pragma unroll
                    for (int i = 0; i < kRows; ++i)
#pragma unroll
                        for (int p = 0; p < NP; ++p)
                            y[i][p] = silu2(y[i][p]);
                }
                if (do_res) {
#pragma unroll
                    for (int i = 0; i < kRows; ++i)
#pragma unroll
                        for (int p = 0; p < NP; ++p)
                            y[i][p] = __fadd2_rn(y[i][p],
                                                 make_float2(xv[i][2 * p], xv[i][2 * p + 1]));
                }
#pragma unroll
                for (int i = 0; i < kRows; ++i) {
                    const int64_t t = tg + i;
                    if (!fast && (i >= nb || t < ta))
                        continue;
                    const int64_t off = t * a.C + (int64_t)m * a.G;
                    float o[CH];
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        o[2 * p] = y[i][p].x;
                        o[2 * p + 1] = y[i][p].y;
                    }
#pragma unroll
                    for (int q = 0; q < NV; ++q) {
                        uint32_t w[OB / 4];
                        Elem<OT>::template pack<EV>(&o[q * EV], w);
                        store_words<OB>(
                            out + (off + (int64_t)(tid + q * a.nth) * EV) * sizeof(OT), w);
                    }
                }
                nslot += nb;
                if (nslot >= a.norm_slots)
                    nslot -= a.norm_slots;
            }
        }
        // inv_s / nv_s of this buffer are rewritten two chunks later, after
        // the next chunk's barrier: no second barrier needed
    }
}

} // namespace ple
} // namespace engram
