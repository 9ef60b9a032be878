// ple_conv_bwd.cuh -- backward of the PLE tail of ple_conv.cuh (engram page,
// Qwen3_8_FlashNextPLELayer: norm_conv, conv1d, _causal_short_conv; layers
// page, Qwen3_8_FlashNextGroupedRMSNorm), for training the layer.
//
// Forward, per branch slice of G features and token t (s = 1 + norm_w):
//   xh = x * inv,  inv = rsqrt(mean(x^2) + eps);   n = s * xh
//   y  = bias + sum_{k <= back(t)} w_k n[t - k d],  w_k = conv_w[K-1-k]
//   out = x + SiLU(y)
// Backward, given dout:
//   dy = dout * SiLU'(y),  SiLU'(y) = sg (1 + y (1 - sg)),  sg = sigmoid(y)
//   dn[t] = sum_{k <= fwd(t)} w_k dy[t + k d]       (transposed convolution)
//   dx = inv (s dn - xh mean_G(s dn xh)) + dout
//   dbias = sum_t dy,  dconv_w[K-1-k] = s sum_t dy[t + k d] xh[t],
//   dnorm_w = sum_t dn xh
// where back(t) / fwd(t) count the taps that stay inside t's sequence.
//
// The convolution only couples rows of one residue modulo d, so a block owns
// one branch, one residue r and a range [ja, jb) of that residue's rows
// j (token t = r + j d): along them the convolution has dilation 1. It walks
// the rows in batches of B = 4, with the kernel width fixed at 4 (narrower
// kernels run with zero taps) so that the lag of the transposed convolution
// is 3 rows:
//   stage 1  every thread sums the squares of its 8 channels of the batch's
//            rows (one warp sum for four rows), warps post partial sums;
//   barrier
//   stage 2  inverse RMS of the four rows; y from the rows' normalised
//            history (read again from shared memory), dy into a register
//            ring holding rows j0 - 3 .. j0 + 3;
//   stage 3  for the lagged rows j0 - 3 .. j0: dn from the ring, the weight
//            gradients, and per-warp partials of sum(s dn xh);
//   barrier
//   stage 4  dx of the lagged rows (streaming stores), then the ring shifts.
// Rows reach shared memory through a ring of row slots filled by cp.async.bulk
// (one copy per row of x and of dout, issued `ahead` batches early by thread
// 0, completion on a per-batch mbarrier waited on with a time bound). Halo
// rows (3 before ja for history, 3 after jb for dy) are read but own no
// output. Each block writes its weight-gradient partials to a workspace,
// [d * chunks][4 + 2][C] fp32, that conv_bwd_reduce_kernel sums in a fixed
// order, so results do not depend on timing.
#pragma once

#include "ple_conv_reg.cuh"

namespace engram {
namespace ple {

constexpr int kBwdRows = 4;                    // rows per batch
constexpr int kBwdTaps = 4;                    // kernel widths 1..4
constexpr int kBwdLag = kBwdTaps - 1;
constexpr int kBwdWarps = 10;                  // 8 channels per thread: G <= 2560
constexpr int kBwdThreads = 32 * kBwdWarps;
constexpr int kBwdPartStride = 12;             // per-row partials, padded for float4 reads
constexpr int kBwdMaxSlots = 32;
constexpr int kBwdBars = 8;
constexpr int kBwdQuantities = kBwdTaps + 2;   // weight taps, bias, norm scale

// Shared memory: square-sum and dot partials [B][12] float each, inverse RMS
// [32] float and tap counts [32] int32 per row slot, mbarriers [8]; then the
// row slots of x [slots][pitch_x] and of dout [slots][pitch_g].
constexpr int kBwdOffDot = kBwdRows * kBwdPartStride * 4;
constexpr int kBwdOffInv = 2 * kBwdOffDot;
constexpr int kBwdOffMeta = kBwdOffInv + kBwdMaxSlots * 4;
constexpr int kBwdOffBars = kBwdOffMeta + kBwdMaxSlots * 4;
constexpr int kBwdHeader = kBwdOffBars + kBwdBars * 8;
constexpr int kBwdDataOffset = (kBwdHeader + 127) / 128 * 128;

__host__ __device__ constexpr size_t bwd_smem_bytes(int slots, int pitch_x, int pitch_g)
{
    return (size_t)kBwdDataOffset + (size_t)slots * (pitch_x + pitch_g);
}

struct ConvBwdArgs {
    const void *x, *dout;
    void *dx;
    float *partial;         // [d * chunks][kBwdQuantities][C]
    const int32_t *cu;
    int32_t nseq;
    int64_t T;
    int32_t C, G, nth;      // nth = G / 8 active threads
    int32_t dil, K, chunks; // chunks: blocks per (branch, residue)
    const void *norm_w, *conv_w, *bias;
    int32_t wdtype;
    float eps, inv_G;
    uint32_t flags;
    int32_t slots, ahead;   // row slots; batches in flight ahead of the current one
    int32_t pitch_x, pitch_g;
};

// 8 channels of one row in a shared-memory slot, as floats.
template <typename T>
__device__ __forceinline__ void load_slot8(const unsigned char *p, float *f)
{
    constexpr int W = 8 * (int)sizeof(T) / 4;
    uint32_t w[W];
#pragma unroll
    for (int q = 0; q < W / 4; ++q) {
        const uint4 u = reinterpret_cast<const uint4 *>(p)[q];
        w[4 * q] = u.x;
        w[4 * q + 1] = u.y;
        w[4 * q + 2] = u.z;
        w[4 * q + 3] = u.w;
    }
    Elem<T>::template unpack<8>(w, f);
}

// sum over 12 padded per-warp partials of row i
__device__ __forceinline__ float sum_parts(const float *part, int i)
{
    const float4 *p = reinterpret_cast<const float4 *>(part + i * kBwdPartStride);
    const float4 a = p[0], b = p[1], c = p[2];
    return ((a.x + a.y) + (a.z + a.w)) + ((b.x + b.y) + (b.z + b.w)) +
           ((c.x + c.y) + (c.z + c.w));
}

template <typename XT, typename GT>
__global__ void __launch_bounds__(kBwdThreads, 1) short_conv_bwd_kernel(const ConvBwdArgs a)
{
    constexpr int B = kBwdRows, L = kBwdLag, KT = kBwdTaps, CH = 8, NP = CH / 2;
    constexpr int RING = L + B;
    extern __shared__ __align__(128) unsigned char smem[];
    float *ss_part = reinterpret_cast<float *>(smem);
    float *dot_part = reinterpret_cast<float *>(smem + kBwdOffDot);
    float *inv_s = reinterpret_cast<float *>(smem + kBwdOffInv);
    int32_t *meta_s = reinterpret_cast<int32_t *>(smem + kBwdOffMeta);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBwdOffBars);
    unsigned char *xs = smem + kBwdDataOffset;
    unsigned char *gs = xs + (size_t)a.slots * a.pitch_x;

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const bool active = tid < a.nth;
    const int d = a.dil;
    const int per_branch = d * a.chunks;
    const int m = blockIdx.x / per_branch;
    const int rem = blockIdx.x - m * per_branch;
    const int r = rem / a.chunks, p = rem - r * a.chunks;
    const int64_t nr = a.T > r ? (a.T - r + d - 1) / d : 0;  // rows of residue r
    const int64_t ja = nr * p / a.chunks, jb = nr * (p + 1) / a.chunks;
    const int64_t c0 = (int64_t)m * a.G + (int64_t)tid * CH;  // first channel of this thread
    float *part = a.partial + (size_t)(r * a.chunks + p) * kBwdQuantities * a.C + c0;

    if (ja >= jb) {  // no rows: the block's partials are zero
        if (active)
#pragma unroll
            for (int q = 0; q < kBwdQuantities; ++q) {
                reinterpret_cast<float4 *>(part + (size_t)q * a.C)[0] = make_float4(0, 0, 0, 0);
                reinterpret_cast<float4 *>(part + (size_t)q * a.C)[1] = make_float4(0, 0, 0, 0);
            }
        return;
    }
    const int64_t js = ja - L > 0 ? ja - L : 0;
    const int64_t je = min64(nr, jb + L);
    const int nbatch = (int)((jb + L - js + B - 1) / B);
    const int S = a.slots;
    const uint32_t xbytes = (uint32_t)a.G * sizeof(XT), gbytes = (uint32_t)a.G * sizeof(GT);
    const char *xb = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    const char *gb = static_cast<const char *>(a.dout) + (int64_t)m * a.G * sizeof(GT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT), grow = (int64_t)a.C * sizeof(GT);
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;

    // sequence frontier of the loading thread: [seq_lo, seq_hi) holds the
    // last row it described
    int32_t seq = 0;
    int64_t seq_lo = 0, seq_hi = a.T;
    if (tid == 0) {
        for (int b = 0; b < kBwdBars; ++b)
            mbar_init(bars + b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (a.cu != nullptr) {
            seq = find_sequence(a.cu, a.nseq, r + js * d);
            seq_lo = __ldg(a.cu + seq);
            seq_hi = __ldg(a.cu + seq + 1);
        }
    }
    for (int i = tid; i < 2 * B * kBwdPartStride; i += blockDim.x)
        ss_part[i] = 0.f;  // (and dot_part) pads of absent warps stay zero
    for (int i = tid; i < kBwdMaxSlots; i += blockDim.x) {
        inv_s[i] = 0.f;
        meta_s[i] = 0;
    }
    __syncthreads();

    // thread 0: rows of batch b into their slots, and their tap counts
    auto issue = [&](int b) {
        const int64_t j0 = js + (int64_t)b * B;
        uint32_t bytes = 0;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int64_t j = j0 + i;
            if (j < je)
                bytes += xbytes + (j >= ja ? gbytes : 0u);
        }
        if (bytes == 0)
            return;
        uint64_t *bar = bars + b % kBwdBars;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                     "r"(bytes)
                     : "memory");
        int slot = (int)((j0 - js) % S);
#pragma unroll
        for (int i = 0; i < B; ++i, slot = slot + 1 == S ? 0 : slot + 1) {
            const int64_t j = j0 + i;
            if (j >= je)
                break;
            const int64_t t = r + j * d;
            bulk_load(xs + (size_t)slot * a.pitch_x, xb + t * xrow, xbytes, bar);
            if (j >= ja)
                bulk_load(gs + (size_t)slot * a.pitch_g, gb + t * grow, gbytes, bar);
            if (a.cu != nullptr)
                while (t >= seq_hi && seq + 1 < a.nseq) {
                    ++seq;
                    seq_lo = seq_hi;
                    seq_hi = __ldg(a.cu + seq + 1);
                }
            const int64_t back = (t - seq_lo) / d, fwd = (seq_hi - 1 - t) / d;
            const int nb = back <= 0 ? 0 : back >= L ? L : (int)back;
            const int nf = fwd <= 0 ? 0 : fwd >= L ? L : (int)fwd;
            meta_s[slot] = nb | nf << 8;
        }
    };
    if (tid == 0)
        for (int b = 0; b < a.ahead && b < nbatch; ++b)
            issue(b);

    // this thread's weights, norm scale and bias, in channel pairs
    float2 w[KT][NP], sc[NP], bias[NP];
#pragma unroll
    for (int e = 0; e < CH; ++e) {
        const int64_t c = c0 + e;
        const float s =
            active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
        const float bv = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
        (e & 1 ? sc[e / 2].y : sc[e / 2].x) = s;
        (e & 1 ? bias[e / 2].y : bias[e / 2].x) = bv;
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            const float wv =
                active && k < a.K ? load_weight(a.conv_w, a.wdtype, c * a.K + (a.K - 1 - k)) : 0.f;
            (e & 1 ? w[k][e / 2].y : w[k][e / 2].x) = wv;
        }
    }
    const float2 zero2 = make_float2(0.f, 0.f);
    float2 dy[RING][NP];  // rows j0 - L .. j0 + B - 1 of the current batch
    float2 dw[KT][NP], db[NP], dnw[NP];
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
#pragma unroll
        for (int i = 0; i < RING; ++i)
            dy[i][pp] = zero2;
#pragma unroll
        for (int k = 0; k < KT; ++k)
            dw[k][pp] = zero2;
        db[pp] = zero2;
        dnw[pp] = zero2;
    }

    const size_t xoff = (size_t)tid * CH * sizeof(XT), goff = (size_t)tid * CH * sizeof(GT);
    char *dxb = static_cast<char *>(a.dx) + (int64_t)m * a.G * sizeof(GT) + goff;
    bool timed_out = false;

    for (int b = 0; b < nbatch; ++b) {
        const int64_t j0 = js + (int64_t)b * B;
        int slot[B];
        slot[0] = (int)((j0 - js) % S);
#pragma unroll
        for (int i = 1; i < B; ++i)
            slot[i] = slot[i - 1] + 1 == S ? 0 : slot[i - 1] + 1;
        if (j0 < je && !timed_out &&
            !mbar_wait(bars + b % kBwdBars, (uint32_t)(b / kBwdBars) & 1u))
            timed_out = true;

        // ---- stage 1: squares of the batch's rows
        if (do_norm) {
            float ss[B];
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float2 acc = zero2;
                if (active && j0 + i < je) {
                    float f[CH];
                    load_slot8<XT>(xs + (size_t)slot[i] * a.pitch_x + xoff, f);
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp) {
                        const float2 x2 = make_float2(f[2 * pp], f[2 * pp + 1]);
                        acc = __ffma2_rn(x2, x2, acc);
                    }
                }
                ss[i] = acc.x + acc.y;
            }
            const float tot = warp_sum4(ss[0], ss[1], ss[2], ss[3], lane);
            if ((lane & 7) == 0)
                ss_part[(lane >> 3) * kBwdPartStride + wid] = tot;
        }
        __syncthreads();
        if (tid == 0 && b + a.ahead < nbatch)
            issue(b + a.ahead);

        // ---- stage 2: inverse RMS, y and dy of the batch's rows
        float inv[B];
#pragma unroll
        for (int i = 0; i < B; ++i) {
            inv[i] = do_norm ? rsqrtf(fmaf(sum_parts(ss_part, i), a.inv_G, a.eps)) : 1.f;
            if (tid == 0)
                inv_s[slot[i]] = inv[i];
        }
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int64_t j = j0 + i;
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                dy[L + i][pp] = zero2;
            if (!active || j >= je || j < ja)
                continue;
            const int back = meta_s[slot[i]] & 0xff;
            float2 acc[NP];
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                acc[pp] = zero2;
#pragma unroll
            for (int k = 0; k < KT; ++k) {
                if (k > back)
                    break;
                const int sk = slot[i] - k < 0 ? slot[i] - k + S : slot[i] - k;
                const float ik = i - k >= 0 ? inv[i - k >= 0 ? i - k : 0] : inv_s[sk];
                float f[CH];
                load_slot8<XT>(xs + (size_t)sk * a.pitch_x + xoff, f);
                const float2 ik2 = make_float2(ik, ik);
#pragma unroll
                for (int pp = 0; pp < NP; ++pp)
                    acc[pp] = __ffma2_rn(
                        w[k][pp], __fmul2_rn(make_float2(f[2 * pp], f[2 * pp + 1]), ik2), acc[pp]);
            }
            float g[CH];
            load_slot8<GT>(gs + (size_t)slot[i] * a.pitch_g + goff, g);
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                const float2 y = __ffma2_rn(sc[pp], acc[pp], bias[pp]);
                float2 f = make_float2(1.f, 1.f);
                if (do_silu) {
                    // SiLU'(y) = sg + y sg (1 - sg), sg = 1 / (1 + 2^(-y log2 e))
                    constexpr float kNegLog2e = -1.4426950408889634f;
                    const float2 z = __fmul2_rn(y, make_float2(kNegLog2e, kNegLog2e));
                    const float2 den = __fadd2_rn(make_float2(ex2_approx(z.x), ex2_approx(z.y)),
                                                  make_float2(1.f, 1.f));
                    const float2 sg = make_float2(rcp_approx(den.x), rcp_approx(den.y));
                    const float2 om = __ffma2_rn(sg, make_float2(-1.f, -1.f),
                                                 make_float2(1.f, 1.f));
                    f = __ffma2_rn(y, __fmul2_rn(sg, om), sg);
                }
                dy[L + i][pp] = __fmul2_rn(make_float2(g[2 * pp], g[2 * pp + 1]), f);
            }
        }

        // ---- stage 3: dn, weight gradients and dot partials of the lagged rows
        {
            float dotv[B];
#pragma unroll
            for (int i = 0; i < B; ++i) {
                const int64_t jj = j0 - L + i;
                float2 acc = zero2;
                if (active && jj >= ja && jj < jb) {
                    const int sl = slot[i] - L < 0 ? slot[i] - L + S : slot[i] - L;
                    const int fwd = meta_s[sl] >> 8;
                    const float ij = i - L >= 0 ? inv[i - L >= 0 ? i - L : 0] : inv_s[sl];
                    float f[CH];
                    load_slot8<XT>(xs + (size_t)sl * a.pitch_x + xoff, f);
                    const float2 ij2 = make_float2(ij, ij);
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp) {
                        const float2 xh = __fmul2_rn(make_float2(f[2 * pp], f[2 * pp + 1]), ij2);
                        float2 dn = zero2;
#pragma unroll
                        for (int k = 0; k < KT; ++k) {
                            const float2 g = k <= fwd ? dy[i + k][pp] : zero2;
                            dn = __ffma2_rn(w[k][pp], g, dn);
                            dw[k][pp] = __ffma2_rn(xh, g, dw[k][pp]);
                        }
                        db[pp] = __fadd2_rn(db[pp], dy[i][pp]);
                        dnw[pp] = __ffma2_rn(dn, xh, dnw[pp]);
                        acc = __ffma2_rn(__fmul2_rn(sc[pp], dn), xh, acc);
                    }
                }
                dotv[i] = acc.x + acc.y;
            }
            if (do_norm) {
                const float tot = warp_sum4(dotv[0], dotv[1], dotv[2], dotv[3], lane);
                if ((lane & 7) == 0)
                    dot_part[(lane >> 3) * kBwdPartStride + wid] = tot;
            }
        }
        __syncthreads();

        // ---- stage 4: dx of the lagged rows
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int64_t jj = j0 - L + i;
            if (!active || jj < ja || jj >= jb)
                continue;
            const int sl = slot[i] - L < 0 ? slot[i] - L + S : slot[i] - L;
            const int fwd = meta_s[sl] >> 8;
            const float ij = i - L >= 0 ? inv[i - L >= 0 ? i - L : 0] : inv_s[sl];
            const float mean = do_norm ? sum_parts(dot_part, i) * a.inv_G : 0.f;
            float f[CH], g[CH], o[CH];
            load_slot8<XT>(xs + (size_t)sl * a.pitch_x + xoff, f);
            if (do_res)
                load_slot8<GT>(gs + (size_t)sl * a.pitch_g + goff, g);
            const float2 ij2 = make_float2(ij, ij), mean2 = make_float2(-mean, -mean);
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                float2 dn = zero2;
#pragma unroll
                for (int k = 0; k < KT; ++k)
                    dn = __ffma2_rn(w[k][pp], k <= fwd ? dy[i + k][pp] : zero2, dn);
                float2 v;
                if (do_norm) {
                    const float2 xh = __fmul2_rn(make_float2(f[2 * pp], f[2 * pp + 1]), ij2);
                    v = __fmul2_rn(ij2, __ffma2_rn(xh, mean2, __fmul2_rn(sc[pp], dn)));
                } else {
                    v = dn;
                }
                if (do_res)
                    v = __fadd2_rn(v, make_float2(g[2 * pp], g[2 * pp + 1]));
                o[2 * pp] = v.x;
                o[2 * pp + 1] = v.y;
            }
            constexpr int OW = CH * (int)sizeof(GT) / 4;
            uint32_t ow[OW];
            Elem<GT>::template pack<CH>(o, ow);
            const int64_t t = r + jj * d;
            store_words<OW * 4>(dxb + t * grow, ow);
        }
        // the ring moves on by one batch
#pragma unroll
        for (int i = 0; i < L; ++i)
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                dy[i][pp] = dy[i + B][pp];
    }

    // partials of this block: s * dw per tap, dbias, dnorm_w (zero without the norm)
    if (active) {
        auto put = [&](int q, const float2 *v) {
            float4 *dst = reinterpret_cast<float4 *>(part + (size_t)q * a.C);
            dst[0] = make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
            dst[1] = make_float4(v[2].x, v[2].y, v[3].x, v[3].y);
        };
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            float2 v[NP];
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                v[pp] = __fmul2_rn(sc[pp], dw[k][pp]);
            put(k, v);
        }
        put(KT, db);
        if (!do_norm)
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                dnw[pp] = zero2;
        put(KT + 1, dnw);
    }
    if (timed_out && lane == 0)
        raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
}

// Sums the blocks' partials in block order (fp64) into the weight gradients:
// dconv_w [C, K] (tap k of the partials is column K-1-k), dbias [C],
// dnorm_w [C]; null outputs are skipped.
__global__ void __launch_bounds__(256) conv_bwd_reduce_kernel(const float *partial, int npart,
                                                              int C, int K, float *dconv_w,
                                                              float *dbias, float *dnorm_w)
{
    const int64_t total = (int64_t)kBwdQuantities * C;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int q = (int)(e / C);
        const int c = (int)(e - (int64_t)q * C);
        float *dst = q < kBwdTaps ? (q < K ? dconv_w + (int64_t)c * K + (K - 1 - q) : nullptr)
                     : q == kBwdTaps ? (dbias ? dbias + c : nullptr)
                                     : (dnorm_w ? dnorm_w + c : nullptr);
        if (dst == nullptr)
            continue;
        double s = 0.0;
        for (int i = 0; i < npart; ++i)
            s += (double)__ldg(partial + ((int64_t)i * kBwdQuantities + q) * C + c);
        *dst = (float)s;
    }
}

} // namespace ple
} // namespace engram
