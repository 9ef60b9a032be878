// ple_conv_cls.cuh -- the PLE tail of ple_conv.cuh (engram page,
// Qwen3_8_FlashNextPLELayer: norm_conv, conv1d, _causal_short_conv; layers
// page, Qwen3_8_FlashNextGroupedRMSNorm) for kernel widths up to 4 and any
// dilation d, one residue class at a time.
//
// The taps of token t read tokens t - d, t - 2d, t - 3d: all of t's residue
// modulo d. A unit of work is one branch, one residue r and a range of that
// residue's rows j (token t = r + j d); along them the convolution has
// dilation 1, so a thread keeps only the last three normalised values of its
// channels. With 4 channels per thread that is 12 registers of history, and a
// 2,560-wide branch takes 20 conv warps -- with the four row-statistics
// warps, 24 warps per SM at 80 registers (a scheduler holds 6 warps, and
// 6 x 32 x 80 fits its 16,384 registers), twice the warps of a design that
// keeps the history of every residue.
//
// Rows travel a batch of 8 at a time through a ring of shared-memory buffers:
//   - stat warps (4): lane i of stat warp 0 moves row i of a batch into its
//     buffer with cp.async.bulk (completion on the buffer's mbarrier); the
//     warps then compute each row's inverse RMS from shared memory (one warp
//     per row, two rows each per batch; with two warps they were the
//     bottleneck) and stat warp 1 the rows' counts of in-sequence taps; each
//     arrives on "described";
//   - conv warps (G / 4 threads): wait on "described", normalise, convolve,
//     apply SiLU and the residual, store 8 bytes per thread and row with
//     streaming stores, then arrive on "consumed" -- the loader waits on it
//     before it reuses the buffer.
// No barrier spans the block inside the loop, so conv warps drift apart by up
// to the ring depth. Every wait is bounded in time: one that runs out raises
// ENGRAM_DEVERR_COPY_TIMEOUT and the thread skips its later waits on other
// warps (not those on its own copies, which it always waits for before the
// block ends), so the kernel always ends promptly. Waits on other warps are
// bounded by ConvArgs::cross_wait_ns, waits on copies by kCopyWaitNs.
// The 3 rows before a range are read for history only.
#pragma once

#include "async_copy.cuh"
#include "ple_conv.cuh"

namespace engram {
namespace ple {

constexpr int kClsTaps = 4;                // kernel widths 1..4 (narrower: zero taps)
constexpr int kClsHist = kClsTaps - 1;
constexpr int kClsRows = 8;                // rows per batch
constexpr int kClsStatWarps = 4;
constexpr int kClsMaxConvWarps = 20;       // 4 channels per thread: G <= 2560
constexpr int kClsMaxBufs = 6;

// Shared memory: inverse RMS [6][8] float, tap counts [6][8] int32, fast
// flags [6] int32, and three mbarriers per buffer; then the row buffers
// [bufs][8][pitch].
constexpr int kClsOffNv = kClsMaxBufs * kClsRows * 4;
constexpr int kClsOffFast = 2 * kClsOffNv;
constexpr int kClsOffBars = (kClsOffFast + kClsMaxBufs * 4 + 7) / 8 * 8;
constexpr int kClsHeader = kClsOffBars + 3 * kClsMaxBufs * 8;
constexpr int kClsDataOffset = (kClsHeader + 127) / 128 * 128;

__host__ __device__ constexpr size_t cls_smem_bytes(int bufs, int pitch)
{
    return (size_t)kClsDataOffset + (size_t)bufs * kClsRows * pitch;
}

// N (4 or 8) consecutive elements of T (8, 16 or 32 bytes) at the
// shared-window address `addr`, as floats.
template <typename T, int N>
__device__ __forceinline__ void load_n(uint32_t addr, float *f)
{
    constexpr int W = N * (int)sizeof(T) / 4;
    uint32_t w[W];
    if constexpr (W == 2) {
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
    } else {
#pragma unroll
        for (int q = 0; q < W / 4; ++q)
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(w[4 * q]), "=r"(w[4 * q + 1]), "=r"(w[4 * q + 2]),
                           "=r"(w[4 * q + 3])
                         : "r"(addr + 16u * q));
    }
    Elem<T>::template unpack<N>(w, f);
}

// Number of taps k in 1..3 with k * d <= span (span < 0 counts as 0).
__device__ __forceinline__ int cls_taps_within(int32_t span, int32_t d)
{
    return (span >= d) + (span >= 2 * d) + (span >= 3 * d);
}

// ConvArgs fields used: x, out, cu, nseq, T, C, G, bpg (chunks per residue),
// nth (= G / 4), norm_w, conv_w, bias, wdtype, eps, inv_G, K, dil, flags,
// reg_bufs, pitch, classes (and with SAVE: inv_out, groups); the grid is
// branches x classes x bpg blocks of 32 * (ceil(nth / 32) + 2) threads.
// SAVE: also store every output row's inverse RMS to inv_out.
template <typename XT, typename OT, int CH, bool SAVE>
__global__ void __maxnreg__(CH == 4 ? 80 : 128)
    short_conv_cls_kernel(const ConvArgs a)
{
    constexpr int B = kClsRows, H = kClsHist, NP = CH / 2;
    extern __shared__ __align__(128) unsigned char smem[];
    float *inv_s = reinterpret_cast<float *>(smem);                         // [bufs][8]
    int32_t *nv_s = reinterpret_cast<int32_t *>(smem + kClsOffNv);         // [bufs][8]
    int32_t *fast_s = reinterpret_cast<int32_t *>(smem + kClsOffFast);     // [bufs]
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + kClsOffBars);  // rows landed
    uint64_t *full_bar = tma_bar + kClsMaxBufs;                             // rows described
    uint64_t *empty_bar = full_bar + kClsMaxBufs;                           // rows consumed
    unsigned char *data = smem + kClsDataOffset;

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int ncw = (blockDim.x >> 5) - kClsStatWarps;  // conv warps
    const int d = a.dil;
    const int per_branch = a.classes * a.bpg;
    const int m = blockIdx.x / per_branch;
    const int rem = blockIdx.x - m * per_branch;
    const int r = rem / a.bpg, p = rem - r * a.bpg;
    // row indices fit 32 bits (T < 2^31)
    const int32_t nr = a.T > r ? (int32_t)((a.T - r + d - 1) / d) : 0;  // rows of residue r
    const int32_t ja = (int32_t)((int64_t)nr * p / a.bpg);
    const int32_t jb = (int32_t)((int64_t)nr * (p + 1) / a.bpg);
    if (ja >= jb)
        return;
    const int32_t js = ja - H > 0 ? ja - H : 0;
    const int nbatch = (int)((jb - js + B - 1) / B);
    const int NB = a.reg_bufs;
    const uint32_t row_bytes = (uint32_t)a.G * sizeof(XT);
    const int pitch = a.pitch;
    const char *xbranch = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT);

    if (tid == 0) {
        for (int b = 0; b < NB; ++b) {
            mbar_init(tma_bar + b, 1);
            mbar_init(full_bar + b, kClsStatWarps);
            mbar_init(empty_bar + b, ncw);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    bool timed_out = false;

    if (wid >= ncw) {
        // ================================================== stat warps
        const int sw = wid - ncw;
        const int nvec = (int)(row_bytes / 16);
        constexpr int EV = 16 / (int)sizeof(XT);
        const bool do_norm = a.flags & ENGRAM_CONV_NORM;
        // lane i of stat warp 0 loads row i of batch c into buffer c % NB
        auto load_batch = [&](int c) {
            const int32_t j0 = js + c * B;
            const int rc = min(B, jb - j0);
            const int b = c % NB;
            if (lane == 0)
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                                 smem_u32(tma_bar + b)),
                             "r"((uint32_t)rc * row_bytes)
                             : "memory");
            __syncwarp();
            if (lane < rc)
                bulk_load(data + (size_t)(b * B + lane) * pitch,
                          xbranch + (int64_t)(r + (j0 + lane) * d) * xrow, row_bytes, tma_bar + b);
        };
        // the sequence holding this lane's row, tracked from row to row
        int32_t seq = 0;
        int32_t seq_lo = 0, seq_hi = (int32_t)a.T;
        if (sw == 1 && lane < B && a.cu != nullptr) {
            seq = find_sequence(a.cu, a.nseq, r + min(js + lane, nr - 1) * d);
            seq_lo = __ldg(a.cu + seq);
            seq_hi = __ldg(a.cu + seq + 1);
        }
        if (sw == 0)
            for (int c = 0; c < NB && c < nbatch; ++c)
                load_batch(c);
        for (int c = 0; c < nbatch; ++c) {
            const int b = c % NB;
            const int32_t j0 = js + c * B;
            const int rc = min(B, jb - j0);
            if (!mbar_wait(tma_bar + b, (uint32_t)(c / NB) & 1u))
                timed_out = true;
            const uint32_t buf = smem_u32(data) + (uint32_t)(b * B) * pitch;
            for (int i = sw; i < rc; i += kClsStatWarps) {
                float2 ss[EV / 2];
#pragma unroll
                for (int e = 0; e < EV / 2; ++e)
                    ss[e] = make_float2(0.f, 0.f);
#pragma unroll 5
                for (int v = lane; v < nvec; v += 32) {
                    uint32_t w[4];
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                                 : "r"(buf + (uint32_t)i * pitch + (uint32_t)v * 16u));
                    float f[EV];
                    Elem<XT>::template unpack<EV>(w, f);
#pragma unroll
                    for (int e = 0; e < EV; e += 2) {
                        const float2 x2 = make_float2(f[e], f[e + 1]);
                        ss[e / 2] = __ffma2_rn(x2, x2, ss[e / 2]);
                    }
                }
#pragma unroll
                for (int e = 1; e < EV / 2; ++e)
                    ss[0] = __fadd2_rn(ss[0], ss[e]);
                float tot = ss[0].x + ss[0].y;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    tot += __shfl_xor_sync(kFull, tot, o);
                if (lane == 0) {
                    const float iv = do_norm ? rsqrtf(fmaf(tot, a.inv_G, a.eps)) : 1.f;
                    inv_s[b * B + i] = iv;
                    if (SAVE && j0 + i >= ja)  // (history rows belong to the block before)
                        a.inv_out[(int64_t)(r + (j0 + i) * d) * a.groups + m] = iv;
                }
            }
            if (sw == 1) {
                int nv = 0;
                const int32_t j = j0 + lane;
                if (lane < rc) {
                    const int32_t t = r + j * d;
                    if (a.cu != nullptr)
                        while (t >= seq_hi && seq + 1 < a.nseq) {
                            ++seq;
                            seq_lo = seq_hi;
                            seq_hi = __ldg(a.cu + seq + 1);
                        }
                    nv = cls_taps_within(t - seq_lo, d);
                    nv_s[b * B + lane] = nv;
                }
                const bool row_full = lane >= B || (lane < rc && j >= ja && nv == H);
                const bool full = __all_sync(kFull, row_full);
                if (lane == 0)
                    fast_s[b] = full;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(full_bar + b);
            // the buffer of batch c - 1 takes batch c - 1 + NB once every conv
            // warp is done with it
            if (sw == 0 && c >= 1 && c - 1 + NB < nbatch) {
                const int pb = (c - 1) % NB;
                if (!timed_out && !mbar_wait(empty_bar + pb, (uint32_t)((c - 1) / NB) & 1u,
                                             a.cross_wait_ns))
                    timed_out = true;
                load_batch(c - 1 + NB);
            }
        }
        if (timed_out && lane == 0)
            raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
        return;
    }

    // ====================================================== conv warps
    const bool active = tid < a.nth;
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;
    // weights carry the norm's (1 + w) scale; tap k reads the row k back
    float2 wk[kClsTaps][NP], bias[NP];
#pragma unroll
    for (int e = 0; e < CH; ++e) {
        const int64_t c = (int64_t)m * a.G + (int64_t)tid * CH + e;
        const float scale =
            active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
        const float bv = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
        (e & 1 ? bias[e / 2].y : bias[e / 2].x) = bv;
#pragma unroll
        for (int k = 0; k < kClsTaps; ++k) {
            const float w =
                active && k < a.K ? load_weight(a.conv_w, a.wdtype, c * a.K + (a.K - 1 - k)) * scale
                                  : 0.f;
            (e & 1 ? wk[k][e / 2].y : wk[k][e / 2].x) = w;
        }
    }
    const float2 zero2 = make_float2(0.f, 0.f);
    float2 hist[H][NP];  // normalised values of the last H rows, newest first
#pragma unroll
    for (int h = 0; h < H; ++h)
#pragma unroll
        for (int pp = 0; pp < NP; ++pp)
            hist[h][pp] = zero2;

    char *out = static_cast<char *>(a.out) + ((int64_t)m * a.G + (int64_t)tid * CH) * sizeof(OT);
    const uint32_t xoff = (uint32_t)tid * CH * sizeof(XT);
    const int64_t orow = (int64_t)a.C * sizeof(OT);
    const int64_t ostep = (int64_t)d * orow;  // from one row of the residue to the next
    for (int c = 0; c < nbatch; ++c) {
        const int b = c % NB;
        const int32_t j0 = js + c * B;
        const int rc = min(B, jb - j0);
        if (!timed_out && !mbar_wait(full_bar + b, (uint32_t)(c / NB) & 1u, a.cross_wait_ns))
            timed_out = true;
        const uint32_t buf = smem_u32(data) + (uint32_t)(b * B) * pitch + xoff;
        // the batch's inverse RMS values in two 16-byte loads, and the output
        // row advanced by one stride per row (the conv warps are close to
        // issue-bound, so per-row address and load instructions count)
        static_assert(B == 8, "two float4 of inverse RMS per batch");
        float invb[B];
        {
            const float4 lo = *reinterpret_cast<const float4 *>(inv_s + b * B);
            const float4 hi = *reinterpret_cast<const float4 *>(inv_s + b * B + 4);
            invb[0] = lo.x;
            invb[1] = lo.y;
            invb[2] = lo.z;
            invb[3] = lo.w;
            invb[4] = hi.x;
            invb[5] = hi.y;
            invb[6] = hi.z;
            invb[7] = hi.w;
        }
        char *orow_p = out + (int64_t)(r + j0 * d) * orow;
        auto run = [&](auto fast_tag) {
            constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                if (!FAST && i >= rc)
                    break;
                float xv[CH];
                if (active)
                    load_n<XT, CH>(buf + (uint32_t)i * pitch, xv);
                else
#pragma unroll
                    for (int e = 0; e < CH; ++e)
                        xv[e] = 0.f;
                const float inv = invb[i];
                const float2 inv2 = make_float2(inv, inv);
                int nv = H;
                if constexpr (!FAST)
                    nv = nv_s[b * B + i];
                float2 n[NP], y[NP];
#pragma unroll
                for (int pp = 0; pp < NP; ++pp) {
                    n[pp] = __fmul2_rn(make_float2(xv[2 * pp], xv[2 * pp + 1]), inv2);
                    y[pp] = __ffma2_rn(wk[0][pp], n[pp], bias[pp]);
                }
#pragma unroll
                for (int k = 1; k <= H; ++k)
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp) {
                        float2 h = hist[k - 1][pp];
                        if constexpr (!FAST)
                            h = k <= nv ? h : zero2;
                        y[pp] = __ffma2_rn(wk[k][pp], h, y[pp]);
                    }
#pragma unroll
                for (int pp = 0; pp < NP; ++pp) {
                    hist[2][pp] = hist[1][pp];
                    hist[1][pp] = hist[0][pp];
                    hist[0][pp] = n[pp];
                }
                if (do_silu) {
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp)
                        y[pp] = silu2(y[pp]);
                }
                if (do_res) {
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp)
                        y[pp] = __fadd2_rn(y[pp], make_float2(xv[2 * pp], xv[2 * pp + 1]));
                }
                const int32_t j = j0 + i;
                if (active && (FAST || j >= ja)) {
                    float o[CH];
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp) {
                        o[2 * pp] = y[pp].x;
                        o[2 * pp + 1] = y[pp].y;
                    }
                    constexpr int OW = CH * (int)sizeof(OT) / 4;
                    uint32_t w[OW];
                    Elem<OT>::template pack<CH>(o, w);
                    store_words<OW * 4>(orow_p, w);
                }
                orow_p += ostep;
            }
        };
        // (rc == B keeps the full-batch path inside the block's rows even
        // when a wait on the statistics warps ran out and fast_s is stale)
        if (fast_s[b] && rc == B)
            run(std::true_type{});
        else
            run(std::false_type{});
        __syncwarp();
        if (lane == 0)
            mbar_arrive(empty_bar + b);
    }
    if (timed_out && lane == 0)
        raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
}

} // namespace ple
} // namespace engram
