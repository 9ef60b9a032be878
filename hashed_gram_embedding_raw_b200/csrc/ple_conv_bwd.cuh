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
// The convolution only couples rows of one residue modulo d, so a unit of
// work is one branch, one residue r and a range [ja, jb) of that residue's
// rows j (token t = r + j d): along them the convolution has dilation 1. A
// thread owns 4 channels and keeps their state in registers (the dy ring of 7
// rows, weights, weight-gradient sums: at 8 channels this needed ~250
// registers, five warps per SM), 168 registers at ten warps per block; a
// branch wider than 1,280 channels is split between the two blocks of a
// cluster, which exchange their per-row partial sums through distributed
// shared memory. The unit walks its rows in batches of B = 4,
// with the kernel width fixed at 4 (narrower kernels run with zero taps) so
// that the lag of the transposed convolution is 3 rows:
//   stage 1  every thread sums the squares of its 4 channels of the batch's
//            rows (one warp sum for four rows); warps post partial sums to
//            both blocks;
//   stage 2  inverse RMS of the four rows; every row of the ring (j0 - 3 ..
//            j0 + 3) is read and normalised once and added into the y of the
//            batch rows it is a tap of; dy into a register ring;
//   stage 3  for the lagged rows j0 - 3 .. j0: dn from the ring, the weight
//            gradients, and partials of sum(s dn xh), posted to both blocks;
//   stage 4  dx of the lagged rows (streaming stores), then the ring shifts.
// Stages 1 and 3 post partial sums that stages 2 and 4 need complete; the
// batches are software-pipelined so that one synchronisation serves both:
// iteration b runs stage 4 of batch b - 1, stages 2 and 3 of batch b and
// stage 1 of batch b + 1, then a block barrier and a wait for the partner
// block's posts (asynchronous stores into this block's shared memory that
// complete on an mbarrier), so no cluster-scope release has to wait for the
// dx stores of stage 4.
// Rows whose taps all stay inside their sequence (nearly all) take a path
// without per-tap masks. Rows reach shared memory through a ring of row
// slots filled by cp.async.bulk (one copy per row of x and of dout, issued
// `ahead` batches early by four lanes of warp 0, completion on a per-batch
// mbarrier waited on with a time bound). Halo rows (3 before ja for history,
// 3 after jb for dy) are read but own no output. Each block writes its
// weight-gradient partials to a workspace, [d * chunks][4 + 2][C] fp32, that
// conv_bwd_reduce_kernel sums in a fixed order, so results do not depend on
// timing.
#pragma once

#include "async_copy.cuh"
#include "ple_conv.cuh"

namespace engram {
namespace ple {

constexpr int kBwdRows = 4;                    // rows per batch
constexpr int kBwdTaps = 4;                    // kernel widths 1..4
constexpr int kBwdLag = kBwdTaps - 1;
constexpr int kBwdCtaWarps = 10;               // per block of a cluster
constexpr int kBwdThreads = 32 * kBwdCtaWarps; // 4 channels per thread
constexpr int kBwdMaxCluster = 2;              // blocks sharing a branch: G <= 2560
constexpr int kBwdPartStride = 24;             // per-row partials (20 warps), padded for float4
constexpr int kBwdMaxSlots = 32;
constexpr int kBwdBars = 8;                    // row-copy barriers (batch % 8)
constexpr int kBwdPartBars = 2;                // partner-partial barriers (phase % 2)
constexpr int kBwdQuantities = kBwdTaps + 2;   // weight taps, bias, norm scale

// Shared memory: square-sum and dot partials [2][B][24] float each (by batch
// parity; column rank * 10 + warp; the pads stay zero), tap counts [32] int32
// per row slot, mbarriers [8 + 2]; then the row slots of x [slots][pitch_x] and
// of dout [slots][pitch_g]. With batches in flight from the one being
// finished (its window reaches 3 rows back) to `ahead` past the next,
// slots = 3 + (ahead + 2) * 4.
constexpr int kBwdOffDot = 2 * kBwdRows * kBwdPartStride * 4;  // two buffers each
constexpr int kBwdOffMeta = 2 * kBwdOffDot;
constexpr int kBwdOffBars = kBwdOffMeta + kBwdMaxSlots * 4;
constexpr int kBwdHeader = kBwdOffBars + (kBwdBars + kBwdPartBars) * 8;
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
    int32_t classes;        // residues holding rows, min(dil, T): the grid's residue extent
    const void *norm_w, *conv_w, *bias;
    int32_t wdtype;
    float eps, inv_G;
    uint32_t flags;
    int32_t slots, ahead;   // row slots; batches in flight ahead of the current one
    int32_t pitch_x, pitch_g;
    int32_t csize;          // blocks per cluster sharing one branch slice (1 or 2)
};

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Barrier over every thread of the cluster, ordering shared-memory accesses
// (local and remote) before it against those after it.
__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// A float into the same offset of block `rank`'s shared memory, stored
// asynchronously: the store completes 4 bytes of transaction count on the
// mbarrier at `bar`'s offset in that block, and a thread there that sees the
// barrier's phase complete sees the value. No fence: the storing thread's
// earlier global stores are not waited for.
__device__ __forceinline__ void st_async_cluster(const float *local, uint32_t rank, float v,
                                                 const uint64_t *bar)
{
    uint32_t remote, rbar;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(local)),
                 "r"(rank));
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rbar) : "r"(smem_u32(bar)),
                 "r"(rank));
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.f32 [%0], %1, [%2];" ::"r"(
                     remote),
                 "f"(v), "r"(rbar)
                 : "memory");
}

// 4 channels of one row in a shared-memory slot (8 or 16 bytes at the
// shared-window address `addr`), as floats.
template <typename T>
__device__ __forceinline__ void load_slot4(uint32_t addr, float *f)
{
    uint32_t w[4];
    if constexpr (sizeof(T) == 2)
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
    else
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                     : "r"(addr));
    Elem<T>::template unpack<4>(w, f);
}

// Number of taps k in 1..3 with k * d <= span (span < 0 counts as 0).
__device__ __forceinline__ int taps_within(int32_t span, int32_t d)
{
    return (span >= d) + (span >= 2 * d) + (span >= 3 * d);
}

// The totals of the four rows' padded per-warp partials, in every lane: lane
// l adds columns l % 8, +8, +16 of row l / 8, the eight lanes of a row combine
// by shuffles, and each row's total is broadcast from its first lane.
__device__ __forceinline__ void sum_parts4(const float *part, int lane, float (&tot)[4])
{
    static_assert(kBwdPartStride == 24 && kBwdRows == 4, "lane layout");
    const float *p = part + (lane >> 3) * kBwdPartStride + (lane & 7);
    float v = (p[0] + p[8]) + p[16];
    v += __shfl_xor_sync(kFull, v, 4);
    v += __shfl_xor_sync(kFull, v, 2);
    v += __shfl_xor_sync(kFull, v, 1);
#pragma unroll
    for (int i = 0; i < 4; ++i)
        tot[i] = __shfl_sync(kFull, v, 8 * i);
}

template <typename XT, typename GT>
__global__ void __launch_bounds__(kBwdThreads, 1) short_conv_bwd_kernel(const ConvBwdArgs a)
{
    constexpr int B = kBwdRows, L = kBwdLag, KT = kBwdTaps, CH = 4, NP = CH / 2;
    constexpr int RING = L + B;
    extern __shared__ __align__(128) unsigned char smem[];
    float *ss_part = reinterpret_cast<float *>(smem);
    float *dot_part = reinterpret_cast<float *>(smem + kBwdOffDot);
    int32_t *meta_s = reinterpret_cast<int32_t *>(smem + kBwdOffMeta);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBwdOffBars);
    uint64_t *pbars = bars + kBwdBars;  // the partner's partials of phase k land on pbars[k % 2]
    unsigned char *xs = smem + kBwdDataOffset;
    unsigned char *gs = xs + (size_t)a.slots * a.pitch_x;

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const bool active = tid < a.nth;
    const int d = a.dil;
    const bool pair = a.csize == 2;
    const uint32_t q_cta = pair ? cluster_rank() : 0u;  // half of the branch slice
    const int unit = blockIdx.x / a.csize;
    const int per_branch = a.classes * a.chunks;
    const int m = unit / per_branch;
    const int rem = unit - m * per_branch;
    const int r = rem / a.chunks, p = rem - r * a.chunks;
    // row indices fit 32 bits (T < 2^31)
    const int32_t nr = a.T > r ? (int32_t)((a.T - r + d - 1) / d) : 0;  // rows of residue r
    const int32_t ja = (int32_t)((int64_t)nr * p / a.chunks);
    const int32_t jb = (int32_t)((int64_t)nr * (p + 1) / a.chunks);
    const int gc = a.G / a.csize;                               // channels of this block
    const int64_t cb = (int64_t)m * a.G + (int64_t)q_cta * gc;  // first channel of this block
    const int64_t c0 = cb + (int64_t)tid * CH;                  // first channel of this thread
    float *part = a.partial + (size_t)(r * a.chunks + p) * kBwdQuantities * a.C + c0;
    const int pslot = (int)q_cta * kBwdCtaWarps + wid;         // this warp's partial column

    if (ja >= jb) {  // no rows: the block's partials are zero
        if (active)
#pragma unroll
            for (int q = 0; q < kBwdQuantities; ++q)
                *reinterpret_cast<float4 *>(part + (size_t)q * a.C) = make_float4(0, 0, 0, 0);
        return;
    }
    const int32_t js = ja - L > 0 ? ja - L : 0;
    const int32_t je = min(nr, jb + L);
    const int nbatch = (int)((jb + L - js + B - 1) / B);
    const int S = a.slots;
    const uint32_t xbytes = (uint32_t)gc * sizeof(XT), gbytes = (uint32_t)gc * sizeof(GT);
    const char *xb = static_cast<const char *>(a.x) + cb * sizeof(XT);
    const char *gb = static_cast<const char *>(a.dout) + cb * sizeof(GT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT), grow = (int64_t)a.C * sizeof(GT);
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;

    // warp 0, lane i < B: rows j0 + i of every batch; each such lane keeps
    // the bounds [seq_lo, seq_hi) of the sequence holding its last row
    int32_t seq = 0;
    int32_t seq_lo = 0, seq_hi = (int32_t)a.T;
    if (wid == 0 && lane < B && a.cu != nullptr) {
        const int32_t t = r + min(js + lane, nr - 1) * d;
        seq = find_sequence(a.cu, a.nseq, t);
        seq_lo = __ldg(a.cu + seq);
        seq_hi = __ldg(a.cu + seq + 1);
    }
    if (tid == 0) {
        for (int b = 0; b < kBwdBars + kBwdPartBars; ++b)
            mbar_init(bars + b, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    for (int i = tid; i < 4 * B * kBwdPartStride; i += blockDim.x)
        ss_part[i] = 0.f;  // (and dot_part) pads of absent warps stay zero
    for (int i = tid; i < kBwdMaxSlots; i += blockDim.x)
        meta_s[i] = 0;
    // Partial sums are posted in phases: phase 0 before the batch loop,
    // phase b + 1 in iteration b. Each post is one row sum per warp and row,
    // stored by 4 lanes into this block's partials and, in a pair, into the
    // partner's with asynchronous stores that complete on the partner's
    // pbars[phase % 2].
    bool timed_out = false;  // a bounded wait gave up (the result is then not valid)
    uint32_t phase = 0;
    auto post = [&](float *partials, float tot) {
        if ((lane & 7) == 0) {
            float *dst = partials + (lane >> 3) * kBwdPartStride + pslot;
            *dst = tot;
            if (pair)
                st_async_cluster(dst, q_cta ^ 1u, tot, pbars + (phase & 1));
        }
    };
    // End of a phase with `nposts` posts: this block's partials are complete
    // after a block barrier (which also orders the ring slots for reuse), the
    // partner's once their bytes (4 lanes x 4 B per warp and post) have landed
    // on pbars[phase % 2]; no cluster-scope release, so the global dx stores
    // are not waited for. The double-buffered partials cannot be overwritten
    // early: a block posts phase k + 2 only after the partner's phase k + 1
    // posts, which the partner makes after it has read phase k's.
    auto end_phase = [&](int nposts) {
        if (pair) {
            uint64_t *pb = pbars + (phase & 1);
            if (tid == 0)
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                                 smem_u32(pb)),
                             "r"((uint32_t)nposts * 16u * (blockDim.x >> 5))
                             : "memory");
            __syncthreads();
            if (!timed_out && !mbar_wait(pb, (phase >> 1) & 1u))
                timed_out = true;
        } else {
            __syncthreads();
        }
        ++phase;
    };
    // every block of the cluster has started, initialised its barriers and
    // zeroed its partials before any block writes into another's
    if (pair)
        cluster_barrier();
    else
        __syncthreads();

    // warp 0: rows of batch b (first slot s0) into their slots (lane i: row
    // j0 + i), and their in-sequence tap counts
    const uint32_t xs_u = smem_u32(xs), gs_u = smem_u32(gs);
    auto issue = [&](int b, int s0) {
        const int32_t j0 = js + b * B;
        if (j0 >= je)
            return;
        uint64_t *bar = bars + b % kBwdBars;
        if (lane == 0) {
            uint32_t bytes = 0;
#pragma unroll
            for (int i = 0; i < B; ++i)
                if (j0 + i < je)
                    bytes += xbytes + (j0 + i >= ja ? gbytes : 0u);
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                             smem_u32(bar)),
                         "r"(bytes)
                         : "memory");
        }
        __syncwarp();
        const int32_t j = j0 + lane;
        if (lane < B && j < je) {
            const int slot = s0 + lane >= S ? s0 + lane - S : s0 + lane;
            const int32_t t = r + j * d;
            bulk_load(xs + (size_t)slot * a.pitch_x, xb + (int64_t)t * xrow, xbytes, bar);
            if (j >= ja)
                bulk_load(gs + (size_t)slot * a.pitch_g, gb + (int64_t)t * grow, gbytes, bar);
            if (a.cu != nullptr)
                while (t >= seq_hi && seq + 1 < a.nseq) {
                    ++seq;
                    seq_lo = seq_hi;
                    seq_hi = __ldg(a.cu + seq + 1);
                }
            meta_s[slot] = taps_within(t - seq_lo, d) | taps_within(seq_hi - 1 - t, d) << 8;
        }
    };
    // first slot of batch b + n from that of batch b (n * B < S)
    auto slot_ahead = [&](int s0, int n) {
        const int v = s0 + n * B;
        return v >= S ? v - S : v;
    };
    int s_issue = 0;  // first slot of the next batch to issue
    if (wid == 0)
        for (int b = 0; b < a.ahead && b < nbatch; ++b) {
            issue(b, s_issue);
            s_issue = slot_ahead(s_issue, 1);
        }

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

    const uint32_t xoff = (uint32_t)tid * CH * sizeof(XT), goff = (uint32_t)tid * CH * sizeof(GT);
    const uint32_t xs_t = xs_u + xoff, gs_t = gs_u + goff;  // this thread's channels, slot 0
    const uint32_t px = (uint32_t)a.pitch_x, pg = (uint32_t)a.pitch_g;
    char *dxb = static_cast<char *>(a.dx) + cb * sizeof(GT) + goff;

    // x of ring row q (rows j0 - L .. j0 + B - 1) of the batch, normalised
    auto load_xh = [&](int slot, float iv, float2 *xh) {
        float f[CH];
        load_slot4<XT>(xs_t + (uint32_t)slot * px, f);
        const float2 iv2 = make_float2(iv, iv);
#pragma unroll
        for (int pp = 0; pp < NP; ++pp)
            xh[pp] = __fmul2_rn(make_float2(f[2 * pp], f[2 * pp + 1]), iv2);
    };

    // slots of the ring rows j0 - L .. j0 + B - 1 of the batch whose first
    // row is in slot s0
    auto window_slots = [&](int s0, int (&slot)[RING]) {
        slot[L] = s0;
#pragma unroll
        for (int q = L - 1; q >= 0; --q)
            slot[q] = slot[q + 1] == 0 ? S - 1 : slot[q + 1] - 1;
#pragma unroll
        for (int q = L + 1; q < RING; ++q)
            slot[q] = slot[q - 1] + 1 == S ? 0 : slot[q - 1] + 1;
    };
    constexpr int PB = B * kBwdPartStride;  // one buffer of partials

    // ---- stage 1 of batch b (first slot s0): wait for its rows, post the
    // squares of its rows
    auto stage1 = [&](int b, int s0) {
        const int32_t j0 = js + b * B;
        // (the block's own copies are waited for even after a timeout, so
        // that none is still in flight when the block ends)
        if (j0 < je && !mbar_wait(bars + b % kBwdBars, (uint32_t)(b / kBwdBars) & 1u))
            timed_out = true;
        if (!do_norm)
            return;
        int sl = s0;
        float ss[B];
#pragma unroll
        for (int i = 0; i < B; ++i, sl = sl + 1 == S ? 0 : sl + 1) {
            float2 acc = zero2;
            if (active && j0 + i < je) {
                float f[CH];
                load_slot4<XT>(xs_t + (uint32_t)sl * px, f);
#pragma unroll
                for (int pp = 0; pp < NP; ++pp) {
                    const float2 x2 = make_float2(f[2 * pp], f[2 * pp + 1]);
                    acc = __ffma2_rn(x2, x2, acc);
                }
            }
            ss[i] = acc.x + acc.y;
        }
        post(ss_part + (b & 1) * PB, warp_sum4(ss[0], ss[1], ss[2], ss[3], lane));
    };

    float inv[RING];  // inverse RMS of the ring rows
#pragma unroll
    for (int q = 0; q < RING; ++q)
        inv[q] = 0.f;
    // normalised x of the lagged rows (ring rows 0 .. B - 1), kept from stage
    // 2 of a batch for its stage 3 and, across the barrier, its stage 4
    float2 xl[B][NP];
#pragma unroll
    for (int i = 0; i < B; ++i)
#pragma unroll
        for (int pp = 0; pp < NP; ++pp)
            xl[i][pp] = zero2;

    // ---- stage 4 of batch b (first slot s0): dx of its lagged rows (ring
    // rows 0 .. B - 1), once the dot partials it posted are complete
    auto stage4 = [&](int b, int s0) {
        const int32_t j0 = js + b * B;
        int slot[RING];
        window_slots(s0, slot);
        int fwd[B];
        bool full_fwd = j0 - L >= ja && j0 - L + B <= jb;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            fwd[i] = meta_s[slot[i]] >> 8;
            full_fwd = full_fwd && fwd[i] == L;
        }
        float means[B];
        if (do_norm)
            sum_parts4(dot_part + (b & 1) * PB, lane, means);
        // FAST: every lagged row has its output and all its taps in-sequence
        auto rows = [&](auto fast_tag) {
            constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                const int32_t jj = j0 - L + i;
                if (!FAST && (!active || jj < ja || jj >= jb))
                    continue;
                const float mean = do_norm ? means[i] * a.inv_G : 0.f;
                float g[CH], o[CH];
                const float2 *xh = xl[i];
                if (do_res)
                    load_slot4<GT>(gs_t + (uint32_t)slot[i] * pg, g);
                const float2 ij2 = make_float2(inv[i], inv[i]);
                const float2 mean2 = make_float2(-mean, -mean);
#pragma unroll
                for (int pp = 0; pp < NP; ++pp) {
                    float2 dn = zero2;
#pragma unroll
                    for (int k = 0; k < KT; ++k)
                        if (FAST || k <= fwd[i])
                            dn = __ffma2_rn(w[k][pp], dy[i + k][pp], dn);
                    float2 v = do_norm ? __fmul2_rn(ij2, __ffma2_rn(xh[pp], mean2,
                                                                    __fmul2_rn(sc[pp], dn)))
                                       : dn;
                    if (do_res)
                        v = __fadd2_rn(v, make_float2(g[2 * pp], g[2 * pp + 1]));
                    o[2 * pp] = v.x;
                    o[2 * pp + 1] = v.y;
                }
                constexpr int OW = CH * (int)sizeof(GT) / 4;
                uint32_t ow[OW];
                Elem<GT>::template pack<CH>(o, ow);
                const int32_t t = r + jj * d;
                store_words<OW * 4>(dxb + (int64_t)t * grow, ow);
            }
        };
        if (full_fwd && active)
            rows(std::true_type{});
        else
            rows(std::false_type{});
    };

    // The batches are pipelined so that one barrier separates them: iteration
    // b finishes batch b - 1 (stage 4), computes batch b (stages 2 and 3) and
    // posts the squares of batch b + 1 (stage 1); partials are double-buffered
    // by batch parity, so a warp that runs ahead never overwrites partials
    // another warp still reads.
    stage1(0, 0);
    end_phase(do_norm ? 1 : 0);
    if (wid == 0 && a.ahead < nbatch) {
        issue(a.ahead, s_issue);
        s_issue = slot_ahead(s_issue, 1);
    }
    int s_cur = 0, s_prev = S - B;  // first slots of batches b and b - 1
    for (int b = 0; b < nbatch; ++b) {
        const int32_t j0 = js + b * B;
        if (b > 0) {
            stage4(b - 1, s_prev);
            // the ring moves on by one batch
#pragma unroll
            for (int i = 0; i < L; ++i) {
                inv[i] = inv[i + B];
#pragma unroll
                for (int pp = 0; pp < NP; ++pp)
                    dy[i][pp] = dy[i + B][pp];
            }
        }
        int slot[RING];
        window_slots(s_cur, slot);

        // ---- stage 2: inverse RMS, y and dy of the batch's rows
        {
            float tot[B];
            if (do_norm)
                sum_parts4(ss_part + (b & 1) * PB, lane, tot);
#pragma unroll
            for (int i = 0; i < B; ++i)
                inv[L + i] = do_norm ? rsqrtf(fmaf(tot[i], a.inv_G, a.eps)) : 1.f;
        }
        // taps: a row of the ring feeds rows i = q - L + k of the batch, tap k
        int back[B];
        bool full_back = true;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            back[i] = meta_s[slot[L + i]] & 0xff;
            full_back = full_back && back[i] == L;
        }
        full_back = full_back && j0 + B <= je && j0 >= ja;
        float2 acc[B][NP];
#pragma unroll
        for (int i = 0; i < B; ++i)
#pragma unroll
            for (int pp = 0; pp < NP; ++pp)
                acc[i][pp] = zero2;
        // FAST: every row of the batch has its output and all its taps
        auto taps = [&](auto fast_tag) {
            constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
            for (int q = 0; q < RING; ++q) {
                const int32_t jr = j0 - L + q;
                if (!FAST && (jr < js || jr >= je))
                    continue;  // not loaded (no batch row reads it: its tap is out of range)
                float2 xh[NP];
                load_xh(slot[q], inv[q], xh);
                if (q < B)
#pragma unroll
                    for (int pp = 0; pp < NP; ++pp)
                        xl[q][pp] = xh[pp];
#pragma unroll
                for (int i = 0; i < B; ++i) {
                    const int k = L + i - q;
                    if (k < 0 || k >= KT)
                        continue;
                    if (FAST || k <= back[i]) {
#pragma unroll
                        for (int pp = 0; pp < NP; ++pp)
                            acc[i][pp] = __ffma2_rn(w[k][pp], xh[pp], acc[i][pp]);
                    }
                }
            }
        };
        if (active) {
            if (full_back)
                taps(std::true_type{});
            else
                taps(std::false_type{});
        }
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const int32_t j = j0 + i;
            const bool need = active && j < je && j >= ja;
            float g[CH];
            if (need)
                load_slot4<GT>(gs_t + (uint32_t)slot[L + i] * pg, g);
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) {
                const float2 y = __ffma2_rn(sc[pp], acc[i][pp], bias[pp]);
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
                dy[L + i][pp] = need ? __fmul2_rn(make_float2(g[2 * pp], g[2 * pp + 1]), f)
                                     : zero2;
            }
        }

        // ---- stage 3: dn, weight gradients and dot partials of the lagged rows
        // (ring rows 0 .. B - 1)
        int fwd[B];
        bool full_fwd = j0 - L >= ja && j0 - L + B <= jb;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            fwd[i] = meta_s[slot[i]] >> 8;
            full_fwd = full_fwd && fwd[i] == L;
        }
        {
            float dotv[B];
            // FAST: every lagged row has its output and all its taps in-sequence
            auto rows = [&](auto fast_tag) {
                constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
                for (int i = 0; i < B; ++i) {
                    const int32_t jj = j0 - L + i;
                    float2 accd = zero2;
                    if (FAST || (active && jj >= ja && jj < jb)) {
                        const float2 *xh = xl[i];
#pragma unroll
                        for (int pp = 0; pp < NP; ++pp) {
                            float2 dn = zero2;
#pragma unroll
                            for (int k = 0; k < KT; ++k)
                                if (FAST || k <= fwd[i]) {
                                    dn = __ffma2_rn(w[k][pp], dy[i + k][pp], dn);
                                    dw[k][pp] = __ffma2_rn(xh[pp], dy[i + k][pp], dw[k][pp]);
                                }
                            db[pp] = __fadd2_rn(db[pp], dy[i][pp]);
                            dnw[pp] = __ffma2_rn(dn, xh[pp], dnw[pp]);
                            accd = __ffma2_rn(__fmul2_rn(sc[pp], dn), xh[pp], accd);
                        }
                    }
                    dotv[i] = accd.x + accd.y;
                }
            };
            if (full_fwd && active)
                rows(std::true_type{});
            else
                rows(std::false_type{});
            if (do_norm)
                post(dot_part + (b & 1) * PB,
                     warp_sum4(dotv[0], dotv[1], dotv[2], dotv[3], lane));
        }
        const int s_next = slot_ahead(s_cur, 1);
        if (b + 1 < nbatch)
            stage1(b + 1, s_next);
        end_phase(do_norm ? (b + 1 < nbatch ? 2 : 1) : 0);
        if (wid == 0 && b + 1 + a.ahead < nbatch) {
            issue(b + 1 + a.ahead, s_issue);
            s_issue = slot_ahead(s_issue, 1);
        }
        s_prev = s_cur;
        s_cur = s_next;
    }
    if (nbatch > 0)
        stage4(nbatch - 1, s_prev);

    // partials of this block: s * dw per tap, dbias, dnorm_w (zero without the norm)
    if (active) {
        auto put = [&](int q, const float2 *v) {
            *reinterpret_cast<float4 *>(part + (size_t)q * a.C) =
                make_float4(v[0].x, v[0].y, v[1].x, v[1].y);
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
    // a block leaves only once the partner has received everything it stored
    // into the partner's shared memory
    if (pair)
        cluster_barrier();
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
