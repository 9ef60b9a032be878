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
// range kRows rows at a time:
//   - thread 0 streams each row's branch slice (G * elem contiguous bytes)
//     into a shared-memory ring with cp.async.bulk; every slot completes an
//     mbarrier, and up to raw_slots rows are in flight;
//   - thread v owns 8 channels (one or two 16-byte vectors of the slice). It
//     unpacks them for the step's rows into registers and sums their squares;
//     a warp shuffle plus one __syncthreads_or per step give every thread the
//     slice sums, and after that barrier the step's slots go back to thread 0;
//   - every thread keeps the normalised values of its own channels for the
//     last halo + kRows rows in a private part of shared memory (no other
//     thread reads them, so they need no barrier) and forms the convolution,
//     SiLU and residual for its channels with packed f32x2 arithmetic;
//   - outputs go to global memory with 16-byte streaming stores.
// The halo rows before a block's range are read and normalised but produce no
// output. Waits on the mbarriers are bounded: after kWaitNs the block raises
// ENGRAM_DEVERR_COPY_TIMEOUT, waits (bounded again) for the copies it issued,
// and returns.
#pragma once

#include <cuda_bf16.h>
#include <type_traits>

#include "common.cuh"

namespace engram {
namespace ple {

constexpr int kRows = 4;                 // rows per step
constexpr int kMaxTaps = 8;              // largest kernel width
constexpr int kChan = 8;                 // channels per thread
constexpr int kMaxThreads = 512;         // G <= kMaxThreads * kChan
constexpr int kHeaderBytes = 1152;       // per-step partial sums and row metadata
constexpr int kMinRawSlots = 2 * kRows;  // smallest landing ring
constexpr int kMaxRawSlots = 64;
constexpr size_t kSmemLimit = 227 * 1024;
constexpr uint64_t kWaitNs = 500ull * 1000 * 1000;

struct ConvArgs {
    const void *x;
    void *out;
    const int32_t *cu;
    int32_t nseq;
    int64_t T;
    int32_t C, G;
    int32_t bpg;      // blocks per branch
    int32_t nth;      // active threads per block = G / kChan
    const void *norm_w, *conv_w, *bias;
    int32_t wdtype;
    float eps, inv_G;
    int32_t K, dil, halo;
    int32_t raw_slots, raw_pitch, norm_slots;
    uint32_t flags;   // ENGRAM_CONV_* bits
};

// Bytes before the landing ring: partial sums [2][32] float4, row offsets
// [2][kRows] int64, valid-tap counts [2][kRows] int32, then the mbarriers.
__host__ __device__ constexpr int ring_offset(int raw_slots)
{
    return kHeaderBytes + ((raw_slots * 8 + 127) / 128) * 128;
}

__host__ __device__ constexpr size_t smem_bytes(int raw_slots, int raw_pitch, int norm_slots, int nth)
{
    return (size_t)ring_offset(raw_slots) + (size_t)raw_slots * raw_pitch +
           (size_t)norm_slots * nth * kChan * sizeof(float);
}

// --------------------------------------------------- mbarrier + bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Makes initialised mbarriers visible to the async (bulk copy) proxy.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// One contiguous global -> shared copy by the bulk-copy (TMA) engine; src, dst
// and bytes are multiples of 16. Completion is signalled on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t done;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(done)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for phase `parity` of `bar` to complete; false after kWaitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitNs)
            return false;
    return true;
}

// ------------------------------------------------------ element conversion

template <typename XT>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kPerVec = 4;
    __device__ static void unpack(const uint4 &v, float *f)
    {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerVec = 8;
    // a bf16 value is the upper half of the fp32 with the same bits
    __device__ static void unpack(const uint4 &v, float *f)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static uint32_t pack2(float a, float b)
    {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
};

template <>
struct Elem<__half> {
    static constexpr int kPerVec = 8;
    __device__ static void unpack(const uint4 &v, float *f)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
    __device__ static uint32_t pack2(float a, float b)
    {
        const __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<const uint32_t *>(&h);
    }
};

// Stores n (4 or 8) consecutive outputs of type OT.
template <typename OT, int N>
__device__ __forceinline__ void store_out(OT *p, const float *y)
{
    if constexpr (std::is_same<OT, float>::value) {
#pragma unroll
        for (int q = 0; q < N / 4; ++q)
            st_stream(reinterpret_cast<float4 *>(p) + q,
                      make_float4(y[4 * q], y[4 * q + 1], y[4 * q + 2], y[4 * q + 3]));
    } else {
        static_assert(N == 8, "16-bit outputs are stored 8 at a time");
        uint4 v;
        v.x = Elem<OT>::pack2(y[0], y[1]);
        v.y = Elem<OT>::pack2(y[2], y[3]);
        v.z = Elem<OT>::pack2(y[4], y[5]);
        v.w = Elem<OT>::pack2(y[6], y[7]);
        st_stream(reinterpret_cast<uint4 *>(p), v);
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

// ------------------------------------------------------------------ kernel

// XT: element type of x; OT: of out; KT: kernel width (0 = runtime, <= 8).
template <typename XT, typename OT, int KT>
__global__ void __launch_bounds__(kMaxThreads, 1) short_conv_kernel(const ConvArgs a)
{
    constexpr int EV = Elem<XT>::kPerVec;  // channels per 16-byte vector
    constexpr int NV = kChan / EV;         // vectors per thread (1 or 2)
    constexpr int KM = KT ? KT : kMaxTaps;
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

    float4 *part = reinterpret_cast<float4 *>(smem);                  // [2][32]
    int64_t *meta_off = reinterpret_cast<int64_t *>(smem + 1024);     // [2][kRows]
    int32_t *meta_nv = reinterpret_cast<int32_t *>(smem + 1024 + 64); // [2][kRows]
    uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kHeaderBytes);
    unsigned char *raw = smem + ring_offset(a.raw_slots);
    float4 *nring = reinterpret_cast<float4 *>(raw + (size_t)a.raw_slots * a.raw_pitch);

    // weights of this thread's channels; tap k looks k * dil rows back
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    float2 wk[KM][kChan / 2];
    float bias[kChan];
#pragma unroll
    for (int e = 0; e < kChan; ++e) {
        const int64_t c = (int64_t)m * a.G + (int64_t)(tid + (e / EV) * a.nth) * EV + e % EV;
        const float scale =
            active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
        bias[e] = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
#pragma unroll
        for (int k = 0; k < KM; ++k) {
            float w = 0.f;
            if (active && k < K)
                w = (a.conv_w ? load_weight(a.conv_w, a.wdtype, c * K + (K - 1 - k)) : 1.f) * scale;
            if (e & 1)
                wk[k][e / 2].y = w;
            else
                wk[k][e / 2].x = w;
        }
    }

    if (tid == 0) {
        for (int s = 0; s < a.raw_slots; ++s)
            mbar_init(bar + s, 1);
        mbar_init_fence();
    }
    __syncthreads();

    // producer state (thread 0)
    const uint32_t row_bytes = (uint32_t)a.nth * kChan * sizeof(XT);
    const char *xsrc = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT);
    int64_t next = tlo;
    int next_slot = 0;
    auto issue = [&](int64_t upto) {
        upto = upto < tb ? upto : tb;
        for (; next < upto; ++next) {
            mbar_expect_tx(bar + next_slot, row_bytes);
            bulk_load(raw + (size_t)next_slot * a.raw_pitch, xsrc + next * xrow, row_bytes,
                      bar + next_slot);
            if (++next_slot == a.raw_slots)
                next_slot = 0;
        }
    };
    int32_t cur = 0;  // sequence of the current row (thread 0)
    if (tid == 0) {
        issue(tlo + a.raw_slots);
        if (a.cu != nullptr)
            cur = find_sequence(a.cu, a.nseq, tlo);
    }

    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;
    const unsigned char *my_raw = raw + (size_t)tid * 16;
    OT *out = static_cast<OT *>(a.out);
    int rslot = 0;          // landing slot of the next row to consume
    uint32_t rphase = 0;    // and the parity of its pending phase
    int nslot = 0;          // private-ring slot of the step's first row
    int64_t t0 = tlo;
    int step_slot = 0;
    uint32_t step_phase = 0;
    bool aborted = false;
    for (int64_t step = 0; t0 < tb; t0 += kRows, ++step) {
        const int nb = (int)min64(kRows, tb - t0);
        const int buf = (int)(step & 1);
        step_slot = rslot;
        step_phase = rphase;
        if (tid == 0) {
            for (int i = 0; i < nb; ++i) {
                const int64_t t = t0 + i;
                int64_t start = 0;
                if (a.cu != nullptr) {
                    while (cur + 1 < a.nseq && __ldg(a.cu + cur + 1) <= t)
                        ++cur;
                    start = __ldg(a.cu + cur);
                }
                const int64_t back = t - start;
                meta_nv[buf * kRows + i] =
                    back <= 0 ? 0 : (int)min64(K - 1, (int64_t)((int32_t)back / a.dil));
                meta_off[buf * kRows + i] = t >= ta ? t * a.C + (int64_t)m * a.G : -1;
            }
        }

        // this thread's channels of the step's rows, and their squares
        float xv[kRows][kChan];
        float ss[kRows];
        bool failed = false;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            ss[i] = 0.f;
#pragma unroll
            for (int e = 0; e < kChan; ++e)
                xv[i][e] = 0.f;
            if (i < nb) {
                if (!mbar_wait(bar + rslot, rphase))
                    failed = true;
                else if (active) {
#pragma unroll
                    for (int q = 0; q < NV; ++q) {
                        const uint4 v = *reinterpret_cast<const uint4 *>(
                            my_raw + (size_t)rslot * a.raw_pitch + (size_t)q * a.nth * 16);
                        Elem<XT>::unpack(v, &xv[i][q * EV]);
                    }
#pragma unroll
                    for (int e = 0; e < kChan; ++e)
                        ss[i] = fmaf(xv[i][e], xv[i][e], ss[i]);
                }
                if (++rslot == a.raw_slots) {
                    rslot = 0;
                    rphase ^= 1u;
                }
            }
        }
#pragma unroll
        for (int i = 0; i < kRows; ++i)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                ss[i] += __shfl_xor_sync(kFull, ss[i], o);
        if (lane == 0)
            part[buf * 32 + wid] = make_float4(ss[0], ss[1], ss[2], ss[3]);
        if (__syncthreads_or(failed)) {
            aborted = true;
            break;
        }
        // the step's slots are free again: refill them
        if (tid == 0)
            issue(t0 + nb + a.raw_slots);

        float4 tot = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int w = 0; w < nw; ++w) {
            const float4 p = part[buf * 32 + w];
            tot.x += p.x;
            tot.y += p.y;
            tot.z += p.z;
            tot.w += p.w;
        }
        const float sums[kRows] = {tot.x, tot.y, tot.z, tot.w};

        if (active) {
#pragma unroll
            for (int i = 0; i < kRows; ++i) {
                if (i >= nb)
                    break;
                const float inv = do_norm ? rsqrtf(fmaf(sums[i], a.inv_G, a.eps)) : 1.f;
                const float2 inv2 = make_float2(inv, inv);
                float2 n[kChan / 2];
#pragma unroll
                for (int p = 0; p < kChan / 2; ++p)
                    n[p] = __fmul2_rn(make_float2(xv[i][2 * p], xv[i][2 * p + 1]), inv2);
                int ns = nslot + i;
                if (ns >= a.norm_slots)
                    ns -= a.norm_slots;
                float4 *slot = nring + (size_t)ns * 2 * a.nth + tid;
                slot[0] = make_float4(n[0].x, n[0].y, n[1].x, n[1].y);
                slot[a.nth] = make_float4(n[2].x, n[2].y, n[3].x, n[3].y);

                const int64_t off = meta_off[buf * kRows + i];
                if (off < 0)
                    continue;
                const int nvalid = meta_nv[buf * kRows + i];
                float2 y[kChan / 2];
#pragma unroll
                for (int p = 0; p < kChan / 2; ++p)
                    y[p] = __ffma2_rn(wk[0][p], n[p], make_float2(bias[2 * p], bias[2 * p + 1]));
#pragma unroll
                for (int k = 1; k < KM; ++k) {
                    if (k >= K || k > nvalid)
                        break;
                    int hs = ns - k * a.dil;
                    if (hs < 0)
                        hs += a.norm_slots;
                    const float4 *h = nring + (size_t)hs * 2 * a.nth + tid;
                    const float4 h0 = h[0], h1 = h[a.nth];
                    y[0] = __ffma2_rn(wk[k][0], make_float2(h0.x, h0.y), y[0]);
                    y[1] = __ffma2_rn(wk[k][1], make_float2(h0.z, h0.w), y[1]);
                    y[2] = __ffma2_rn(wk[k][2], make_float2(h1.x, h1.y), y[2]);
                    y[3] = __ffma2_rn(wk[k][3], make_float2(h1.z, h1.w), y[3]);
                }
                float o[kChan];
#pragma unroll
                for (int p = 0; p < kChan / 2; ++p) {
                    o[2 * p] = y[p].x;
                    o[2 * p + 1] = y[p].y;
                }
                if (do_silu) {
#pragma unroll
                    for (int e = 0; e < kChan; ++e)
                        o[e] = __fdividef(o[e], 1.f + __expf(-o[e]));
                }
                if (do_res) {
#pragma unroll
                    for (int e = 0; e < kChan; ++e)
                        o[e] += xv[i][e];
                }
#pragma unroll
                for (int q = 0; q < NV; ++q)
                    store_out<OT, EV>(out + off + (int64_t)(tid + q * a.nth) * EV, &o[q * EV]);
            }
        }
        nslot += kRows;
        if (nslot >= a.norm_slots)
            nslot -= a.norm_slots;
    }

    if (aborted && tid == 0) {
        raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
        // every copy this block issued for rows t0 .. next-1 must land before
        // its shared memory goes away (each wait bounded again)
        int sl = step_slot;
        uint32_t ph = step_phase;
        for (int64_t r = t0; r < next; ++r) {
            mbar_wait(bar + sl, ph);
            if (++sl == a.raw_slots) {
                sl = 0;
                ph ^= 1u;
            }
        }
    }
}

} // namespace ple
} // namespace engram
