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
// thread owns 2 channels, so its state (weights, weight-gradient sums, rings
// of the last four normalised rows and dy rows) fits the registers of 20
// warps per multiprocessor; a branch wider than 1,280 channels is split
// between the 2 blocks of a cluster (among 4 blocks of 640 channels when the
// row slots of 1,280 fp32 channels would not fit shared memory), which
// exchange their per-row partial sums through distributed shared memory.
// The kernel width is fixed at 4
// (narrower kernels run with zero taps), so the transposed convolution lags
// the rows by 3. The unit walks its rows in batches of B = 8:
//   stage 1  every thread sums the squares of its channels of the batch's
//            rows; each warp reduces the eight rows at once and posts one sum
//            per row to every block of the cluster;
//   stage 2  row by row: inverse RMS from the posted sums, the normalised
//            row into a 4-row register ring, y, and dy into a 4-row ring;
//   stage 3  interleaved with stage 2, for the row 3 behind: dn from the dy
//            ring, the weight gradients, the row's partial of sum(s dn xh)
//            (posted like stage 1's) and u = inv s dn + dout, kept in this
//            thread's part of a shared-memory buffer;
//   stage 4  once the sums are complete, dx = u - inv^2 x mean per row
//            (x read again from its row slot), stored with streaming stores.
// Stages 1 and 3 post partial sums that stages 2 and 4 need complete; the
// batches are software-pipelined so that one synchronisation serves both:
// iteration b runs stage 4 of batch b - 1, stages 2 and 3 of batch b and
// stage 1 of batch b + 1, then a block barrier and a wait for the cluster
// partners' posts (asynchronous stores into this block's shared memory that
// complete on an mbarrier; one thread polls it while the others wait at a
// second block barrier), so no cluster-scope release has to wait for the dx
// stores of stage 4.
// Batches whose rows and taps all stay inside their sequence (nearly all)
// take a path without per-tap masks. Rows reach shared memory through rings
// of row slots filled by cp.async.bulk (one copy per row of x and of dout,
// issued `ahead` batches early by eight lanes of the last warp, completion on a
// per-batch mbarrier waited on with a time bound). Halo rows (3 before ja for
// history, 3 after jb for dy) are read but own no output. Each block writes
// its weight-gradient partials to a workspace, [d * chunks][4 + 2][C] fp32,
// that conv_bwd_reduce_kernel sums in a fixed order, so results do not
// depend on timing.
#pragma once

#include "async_copy.cuh"
#include "ple_conv.cuh"

namespace engram {
namespace ple {

constexpr int kBwdRows = 8;                    // rows per batch
constexpr int kBwdTaps = 4;                    // kernel widths 1..4
constexpr int kBwdLag = kBwdTaps - 1;
constexpr int kBwdCh = 2;                      // channels per thread
constexpr int kBwdWarps = 20;                  // warps per block, at most
constexpr int kBwdThreads = 32 * kBwdWarps;
constexpr int kBwdBlockChannels = kBwdCh * kBwdThreads;  // 1280
constexpr int kBwdMaxCluster = 4;              // blocks sharing a branch
constexpr int kBwdCols = 2 * kBwdWarps;        // partial columns per row: blocks x warps
constexpr int kBwdMaxChannels = 2 * kBwdBlockChannels;   // widest branch, 2560
constexpr int kBwdMaxSlots = 64;               // x slots: (ahead + 3) * B, so ahead <= 5
constexpr int kBwdBars = 8;                    // row-copy barriers (batch % 8)
constexpr int kBwdPartBars = 2;                // partner-partial barriers (phase % 2)
constexpr int kBwdQuantities = kBwdTaps + 2;   // weight taps, bias, norm scale
// shared memory for two blocks on one multiprocessor (228 KB, less 1 KB per block)
constexpr size_t kBwdTwoBlockSmem = 112 * 1024;

// Shared memory: square-sum and dot partials [2][B][40] float each (by batch
// parity; column rank * warps + warp, at most 40 columns for 2 blocks of 20
// warps or 4 of 10; columns of absent warps stay zero), tap counts [64] int32
// and inverse RMS [64] float2 per x row slot, the dx coefficients -inv^2 mean
// of the rows stage 4 finishes next [8] float2 (both as equal pairs, ready
// for the packed f32x2 operations), mbarriers [8 + 2]; then u [B][pitch_u] (fp32, each thread its own channels), the x
// ring [(ahead + 3) * B][pitch_x] and the dout ring [(ahead + 2) * B][pitch_g]
// of row slots, B slots per batch. An x row is read until the stage 4 of the
// batch that lags it, a dout row until its stage 3, and batches are issued
// `ahead` past the next one: at an issue the x ring holds the batches from
// the one stage 4 finishes next (3 of its lagged rows are in the batch
// before) to the new one, the dout ring one batch fewer.
constexpr int kBwdPartBytes = 2 * kBwdRows * kBwdCols * 4;  // one kind, both parities
constexpr int kBwdOffDot = kBwdPartBytes;
constexpr int kBwdOffMeta = 2 * kBwdPartBytes;
constexpr int kBwdOffInv = kBwdOffMeta + kBwdMaxSlots * 4;
constexpr int kBwdOffCoef = kBwdOffInv + kBwdMaxSlots * 8;
constexpr int kBwdOffBars = kBwdOffCoef + kBwdRows * 8;
constexpr int kBwdHeader = kBwdOffBars + (kBwdBars + kBwdPartBars) * 8;
constexpr int kBwdDataOffset = (kBwdHeader + 127) / 128 * 128;

__host__ __device__ constexpr size_t bwd_smem_bytes(int ahead, int pitch_x, int pitch_g,
                                                    int pitch_u)
{
    return (size_t)kBwdDataOffset + (size_t)kBwdRows * pitch_u +
           (size_t)kBwdRows * ((ahead + 3) * (size_t)pitch_x + (ahead + 2) * (size_t)pitch_g);
}

struct ConvBwdArgs {
    const void *x, *dout;
    void *dx;
    float *partial;         // [d * chunks][kBwdQuantities][C]
    const int32_t *cu;
    int32_t nseq;
    int64_t T;
    int32_t C, G;
    int32_t gca;            // channels of a cluster's blocks but the last (a multiple of 8)
    int32_t dil, K, chunks; // chunks: units per (branch, residue)
    int32_t classes;        // residues holding rows, min(dil, T): the grid's residue extent
    const void *norm_w, *conv_w, *bias;
    int32_t wdtype;
    float eps, inv_G;
    uint32_t flags;
    int32_t ahead;          // batches in flight ahead of the next one
    int32_t nbx, nbg;       // batches held by the x ring (ahead + 3) and the dout ring (ahead + 2)
    int32_t pitch_x, pitch_g, pitch_u;
    int32_t csize;          // blocks per cluster sharing one branch slice (1, 2 or 4)
    const float *inv_in;    // [T][C / G] inverse RMS saved by the forward, or null
    int32_t groups;         // C / G
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

// The 2 channels of one row at shared-window address `addr` (4 or 8 bytes),
// as floats.
template <typename T>
__device__ __forceinline__ float2 load_pair(uint32_t addr)
{
    uint32_t w[2];
    if constexpr (sizeof(T) == 4)
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr));
    else
        asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(addr));
    float f[2];
    Elem<T>::template unpack<2>(w, f);
    return make_float2(f[0], f[1]);
}

__device__ __forceinline__ float2 load_u(uint32_t addr)
{
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ void store_u(uint32_t addr, float2 v)
{
    asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(v.x), "f"(v.y) : "memory");
}

// 2 channels to global memory with a streaming store.
template <typename T>
__device__ __forceinline__ void store_pair(void *p, float2 v)
{
    if constexpr (sizeof(T) == 4) {
        asm volatile("st.global.cs.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v.x), "f"(v.y)
                     : "memory");
    } else {
        const float f[2] = {v.x, v.y};
        uint32_t w;
        Elem<T>::template pack<2>(f, &w);
        asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(w) : "memory");
    }
}

// Number of taps k in 1..3 with k * d <= span (span < 0 counts as 0).
__device__ __forceinline__ int taps_within(int32_t span, int32_t d)
{
    return (span >= d) + (span >= 2 * d) + (span >= 3 * d);
}

// Sums eight per-lane values over the warp in 9 shuffles (each exchange step
// hands half of the values still held to the partner): lane l ends with the
// total of value l / 4.
__device__ __forceinline__ float warp_sum8(const float (&v)[8], int lane)
{
    const bool h16 = lane & 16;
    float a[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
        a[k] = (h16 ? v[k + 4] : v[k]) + __shfl_xor_sync(kFull, h16 ? v[k] : v[k + 4], 16);
    const bool h8 = lane & 8;
    float b[2];
#pragma unroll
    for (int k = 0; k < 2; ++k)
        b[k] = (h8 ? a[k + 2] : a[k]) + __shfl_xor_sync(kFull, h8 ? a[k] : a[k + 2], 8);
    const bool h4 = lane & 4;
    float c = (h4 ? b[1] : b[0]) + __shfl_xor_sync(kFull, h4 ? b[0] : b[1], 4);
    c += __shfl_xor_sync(kFull, c, 2);
    c += __shfl_xor_sync(kFull, c, 1);
    return c;
}

// The total of row lane / 4 of eight rows' per-warp partials ([8][40],
// columns in a fixed order): lanes 4i..4i+3 add ten columns each of row i and
// combine by shuffles.
__device__ __forceinline__ float row_total8(const float *part, int lane)
{
    static_assert(kBwdCols == 40 && kBwdRows == 8, "lane layout");
    const float *p = part + (lane >> 2) * kBwdCols + (lane & 3);
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < kBwdCols / 4; ++k)
        v += p[4 * k];
    v += __shfl_xor_sync(kFull, v, 1);
    v += __shfl_xor_sync(kFull, v, 2);
    return v;
}

// SiLU'(y) = sg + y sg (1 - sg), sg = 1 / (1 + 2^(-y log2 e)), for a pair.
__device__ __forceinline__ float2 silu_grad2(float2 y)
{
    constexpr float kNegLog2e = -1.4426950408889634f;
    const float2 z = __fmul2_rn(y, make_float2(kNegLog2e, kNegLog2e));
    const float2 den = __fadd2_rn(make_float2(ex2_approx(z.x), ex2_approx(z.y)),
                                  make_float2(1.f, 1.f));
    const float2 sg = make_float2(rcp_approx(den.x), rcp_approx(den.y));
    const float2 om = __ffma2_rn(sg, make_float2(-1.f, -1.f), make_float2(1.f, 1.f));
    return __ffma2_rn(y, __fmul2_rn(sg, om), sg);
}

// WIDE: blocks of 1,280 channels (gca == kBwdBlockChannels), whose slot
// pitches are compile-time constants, so every shared-memory access takes an
// immediate offset.
template <typename XT, typename GT, bool WIDE>
__global__ void __launch_bounds__(kBwdThreads, 1) short_conv_bwd_kernel(const ConvBwdArgs a)
{
    constexpr int B = kBwdRows, L = kBwdLag, KT = kBwdTaps;
    constexpr int PB = B * kBwdCols;  // one buffer of partials
    static_assert(B % 4 == 0 && L < 4 && L < B, "the register rings rotate with the batch");
    extern __shared__ __align__(128) unsigned char smem[];
    float *ss_part = reinterpret_cast<float *>(smem);
    float *dot_part = reinterpret_cast<float *>(smem + kBwdOffDot);
    int32_t *meta_s = reinterpret_cast<int32_t *>(smem + kBwdOffMeta);
    float2 *inv_s = reinterpret_cast<float2 *>(smem + kBwdOffInv);
    float2 *coef_s = reinterpret_cast<float2 *>(smem + kBwdOffCoef);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBwdOffBars);
    uint64_t *pbars = bars + kBwdBars;  // the partners' partials of phase k land on pbars[k % 2]
    unsigned char *us = smem + kBwdDataOffset;
    unsigned char *xs = us + (size_t)B * (WIDE ? kBwdBlockChannels * 4 : a.pitch_u);
    unsigned char *gs =
        xs + (size_t)a.nbx * B * (WIDE ? kBwdBlockChannels * sizeof(XT) : a.pitch_x);

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int d = a.dil;
    const int cs = a.csize;
    const uint32_t q_cta = cs > 1 ? cluster_rank() : 0u;  // part of the branch slice
    const int unit = blockIdx.x / cs;
    const int per_branch = a.classes * a.chunks;
    const int m = unit / per_branch;
    const int rem = unit - m * per_branch;
    const int r = rem / a.chunks, p = rem - r * a.chunks;
    // row indices fit 32 bits (T < 2^31)
    const int32_t nr = a.T > r ? (int32_t)((a.T - r + d - 1) / d) : 0;  // rows of residue r
    const int32_t ja = (int32_t)((int64_t)nr * p / a.chunks);
    const int32_t jb = (int32_t)((int64_t)nr * (p + 1) / a.chunks);
    const int gc = min(a.gca, a.G - (int)q_cta * a.gca);             // channels of this block
    const int64_t cb = (int64_t)m * a.G + (int64_t)q_cta * a.gca;      // first channel of the block
    const int64_t c0 = cb + (int64_t)kBwdCh * tid;                     // first channel of the thread
    const bool active = kBwdCh * tid < gc;
    float *part = a.partial + (size_t)(r * a.chunks + p) * kBwdQuantities * a.C + c0;
    const int nwarps = (int)(blockDim.x >> 5);
    const int pslot = (int)q_cta * nwarps + wid;  // this warp's partial column

    if (ja >= jb) {  // no rows: the block's partials are zero
        if (active)
#pragma unroll
            for (int q = 0; q < kBwdQuantities; ++q)
                *reinterpret_cast<float2 *>(part + (size_t)q * a.C) = make_float2(0.f, 0.f);
        return;
    }
    const int32_t js = ja - L > 0 ? ja - L : 0;
    const int32_t je = min(nr, jb + L);
    const int nbatch = (int)((jb + L - js + B - 1) / B);
    const uint32_t xbytes = (uint32_t)gc * sizeof(XT), gbytes = (uint32_t)gc * sizeof(GT);
    const char *xb = static_cast<const char *>(a.x) + cb * sizeof(XT);
    const char *gb = static_cast<const char *>(a.dout) + cb * sizeof(GT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT), grow = (int64_t)a.C * sizeof(GT);
    const bool do_norm = a.flags & ENGRAM_CONV_NORM;
    const bool do_silu = a.flags & ENGRAM_CONV_SILU;
    const bool do_res = a.flags & ENGRAM_CONV_RESIDUAL;
    // the forward's saved inverse RMS (the norm is on): no squares to sum
    const bool saved = a.inv_in != nullptr;

    // The last warp issues the row copies (warp 0 has the partial sums to add
    // between the barriers): its lane i < B takes rows j0 + i of every batch
    // and keeps the bounds [seq_lo, seq_hi) of the sequence holding its last row
    const int iwarp = nwarps - 1;
    int32_t seq = 0;
    int32_t seq_lo = 0, seq_hi = (int32_t)a.T;
    if (wid == iwarp && lane < B && a.cu != nullptr) {
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
    for (int i = tid; i < 4 * PB; i += blockDim.x)
        ss_part[i] = 0.f;  // (and dot_part) columns of absent warps stay zero
    for (int i = tid; i < kBwdMaxSlots; i += blockDim.x) {
        meta_s[i] = 0;
        inv_s[i] = make_float2(1.f, 1.f);  // stays 1 without the norm
    }
    // Partial sums are posted in phases: phase 0 before the batch loop,
    // phase b + 1 in iteration b. Each post is one row sum per warp and row,
    // stored by 8 lanes into this block's partials and into every partner's
    // with asynchronous stores that complete on the partner's pbars[phase % 2].
    bool timed_out = false;  // a bounded wait gave up (the result is then not valid)
    uint32_t phase = 0;
    auto post = [&](float *partials, float tot) {
        if ((lane & 3) == 0) {
            float *dst = partials + (lane >> 2) * kBwdCols + pslot;
            *dst = tot;
            uint64_t *pb = pbars + (phase & 1);
            if (cs > 1)
                st_async_cluster(dst, q_cta ^ 1u, tot, pb);
            if (cs > 2) {
                st_async_cluster(dst, q_cta ^ 2u, tot, pb);
                st_async_cluster(dst, q_cta ^ 3u, tot, pb);
            }
        }
    };
    // End of a phase whose posts were the squares of batch bs (rows in x
    // slots from xs0) and the dot partials of batch bd (its lagged rows in x
    // slots sd_lo + q for q < 3, sd_hi + q after; either batch absent: -1):
    // this block's partials are complete after a block barrier (which also
    // orders the ring slots for reuse), the partners' once their bytes (8
    // lanes x 4 B per warp, post and partner) have landed on pbars[phase %
    // 2]. Warp 0 waits for those (lane 0 polls), then sums the partials once
    // for the block: the rows' inverse RMS into inv_s by slot, the lagged
    // rows' dx coefficients into coef_s; the others wait at a second barrier,
    // after which they read them. No cluster-scope release, so the global dx stores are not waited
    // for. The double-buffered partials cannot be overwritten early: a block
    // posts phase k + 2 only after every partner's phase k + 1 posts, which
    // each partner makes after its warp 0 has read phase k's.
    auto end_phase = [&](int bs, int xs0, int bd, int sd_lo, int sd_hi) {
        const int nposts = do_norm ? (bs >= 0 && !saved) + (bd >= 0) : 0;
        if (cs > 1 && tid == 0) {
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                             smem_u32(pbars + (phase & 1))),
                         "r"((uint32_t)(nposts * B * 4 * nwarps * (cs - 1)))
                         : "memory");
        }
        __syncthreads();
        if (wid == 0) {
            if (cs > 1) {
                if (lane == 0 && !timed_out && !mbar_wait(pbars + (phase & 1), (phase >> 1) & 1u))
                    timed_out = true;
                __syncwarp();
            }
            if (do_norm && !saved && bs >= 0) {
                const float v = row_total8(ss_part + (bs & 1) * PB, lane);
                if ((lane & 3) == 0) {
                    const float iv = rsqrtf(fmaf(v, a.inv_G, a.eps));
                    inv_s[xs0 + (lane >> 2)] = make_float2(iv, iv);
                }
            }
            if (do_norm && bd >= 0) {
                const float v = row_total8(dot_part + (bd & 1) * PB, lane);
                if ((lane & 3) == 0) {
                    const int q = lane >> 2;
                    const float iv = inv_s[(q < L ? sd_lo : sd_hi) + q].x;
                    const float cf = -(iv * iv) * (v * a.inv_G);
                    coef_s[q] = make_float2(cf, cf);
                }
            }
        }
        __syncthreads();
        ++phase;
    };
    // every block of the cluster has started, initialised its barriers and
    // zeroed its partials before any block writes into another's
    if (cs > 1)
        cluster_barrier();
    else
        __syncthreads();

    // slot pitches
    const uint32_t px = WIDE ? kBwdBlockChannels * sizeof(XT) : (uint32_t)a.pitch_x;
    const uint32_t pg = WIDE ? kBwdBlockChannels * sizeof(GT) : (uint32_t)a.pitch_g;
    const uint32_t pu = WIDE ? kBwdBlockChannels * sizeof(float) : (uint32_t)a.pitch_u;
    // Batch b's rows take the B slots from (b mod nbx) * B of the x ring and
    // from (b mod nbg) * B of the dout ring; tap counts and inverse RMS are
    // kept per x slot. The last warp issues the copies of batch b (lane i: row j0 +
    // i) and notes the rows' in-sequence tap counts.
    // With the saved inverse RMS, lane i also loads row j0 + i's value when it
    // issues the row; the value is stored to the row's slot (as a pair) at
    // once before the loop, and in the loop just before the next iteration's
    // barrier, so the load has an iteration to land and the barrier makes the
    // value visible before the row is computed (at least one batch ahead).
    float inv_pend = 0.f;
    int inv_pend_slot = -1;
    auto store_pending = [&]() {
        if (inv_pend_slot >= 0) {
            inv_s[inv_pend_slot] = make_float2(inv_pend, inv_pend);
            inv_pend_slot = -1;
        }
    };
    auto issue = [&](int b, int xs0, int gs0) {
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
            const int32_t t = r + j * d;
            bulk_load(xs + (size_t)(xs0 + lane) * px, xb + (int64_t)t * xrow, xbytes, bar);
            if (j >= ja)
                bulk_load(gs + (size_t)(gs0 + lane) * pg, gb + (int64_t)t * grow, gbytes, bar);
            if (a.cu != nullptr)
                while (t >= seq_hi && seq + 1 < a.nseq) {
                    ++seq;
                    seq_lo = seq_hi;
                    seq_hi = __ldg(a.cu + seq + 1);
                }
            meta_s[xs0 + lane] = taps_within(t - seq_lo, d) | taps_within(seq_hi - 1 - t, d) << 8;
            if (saved) {
                inv_pend = __ldg(a.inv_in + (int64_t)t * a.groups + m);
                inv_pend_slot = xs0 + lane;
            }
        }
    };
    const int nbx = a.nbx, nbg = a.nbg;
    int ix = 0, ig = 0;  // ring batches of the next batch to issue
    auto issue_next = [&](int b) {
        issue(b, ix * B, ig * B);
        ix = ix + 1 == nbx ? 0 : ix + 1;
        ig = ig + 1 == nbg ? 0 : ig + 1;
    };
    if (wid == iwarp)
        for (int b = 0; b < a.ahead && b < nbatch; ++b) {
            issue_next(b);
            store_pending();
        }

    // this thread's weights, norm scale and bias, as channel pairs
    float2 w[KT], sc, bias;
    {
        float sv[2], bv[2], wv[KT][2];
#pragma unroll
        for (int e = 0; e < kBwdCh; ++e) {
            const int64_t c = c0 + e;
            sv[e] = active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
            bv[e] = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
#pragma unroll
            for (int k = 0; k < KT; ++k)
                wv[k][e] = active && k < a.K
                               ? load_weight(a.conv_w, a.wdtype, c * a.K + (a.K - 1 - k))
                               : 0.f;
        }
        sc = make_float2(sv[0], sv[1]);
        bias = make_float2(bv[0], bv[1]);
#pragma unroll
        for (int k = 0; k < KT; ++k)
            w[k] = make_float2(wv[k][0], wv[k][1]);
    }
    const float2 zero2 = make_float2(0.f, 0.f);
    // rings of the last four rows: normalised x and dy (row j at index j - js mod 4)
    float2 xr[4], dr[4];
    float2 dw[KT], db = zero2, dnw = zero2;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        xr[i] = dr[i] = zero2;
#pragma unroll
    for (int k = 0; k < KT; ++k)
        dw[k] = zero2;

    // shared-window addresses of this thread's channels in slot 0 and in u row 0
    const uint32_t xs_t = smem_u32(xs) + (uint32_t)tid * kBwdCh * sizeof(XT);
    const uint32_t gs_t = smem_u32(gs) + (uint32_t)tid * kBwdCh * sizeof(GT);
    const uint32_t us_t = smem_u32(us) + (uint32_t)tid * sizeof(float2);
    char *dxb = static_cast<char *>(a.dx) + c0 * sizeof(GT);
    const int64_t dstep = (int64_t)d * grow;  // dx bytes from one row of the residue to the next

    // ---- stage 1 of batch b (x ring batch xc): wait for its rows, post the
    // squares of its rows
    auto stage1 = [&](int b, int xc) {
        const int32_t j0 = js + b * B;
        // (the block's own copies are waited for even after a timeout, so
        // that none is still in flight when the block ends)
        if (j0 < je && !mbar_wait(bars + b % kBwdBars, (uint32_t)(b / kBwdBars) & 1u))
            timed_out = true;
        if (!do_norm || saved)
            return;
        const uint32_t xa = xs_t + (uint32_t)(xc * B) * px;
        auto squares = [&](auto all_tag) {
            constexpr bool ALL = decltype(all_tag)::value;  // every row loaded
            float ss[B];
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float v = 0.f;
                if (ALL || (active && j0 + i < je)) {
                    const float2 x = load_pair<XT>(xa + (uint32_t)i * px);
                    v = fmaf(x.x, x.x, x.y * x.y);
                }
                ss[i] = v;
            }
            return warp_sum8(ss, lane);
        };
        const float tot = active && j0 + B <= je ? squares(std::true_type{})
                                                 : squares(std::false_type{});
        post(ss_part + (b & 1) * PB, tot);
    };

    // ---- stage 4 of batch b (x ring batches xc of b, xp of b - 1): dx of its
    // lagged rows j0 - 3 + q, once the dot partials it posted are complete
    auto stage4 = [&](int b, int xc, int xp) {
        const int32_t j0 = js + b * B;
        const int s_lo = xp * B + B - L, s_hi = xc * B - L;  // slot of lagged row q: + q
        auto rows = [&](auto all_tag) {
            constexpr bool ALL = decltype(all_tag)::value;
            // ALL: every lagged row is an output row, from row j0 - 3 on
            char *drow = ALL ? dxb + (int64_t)(r + (j0 - L) * d) * grow : nullptr;
#pragma unroll
            for (int q = 0; q < B; ++q) {
                const int32_t jj = j0 - L + q;
                if (!ALL && (!active || jj < ja || jj >= jb))
                    continue;
                const int sl = (q < L ? s_lo : s_hi) + q;
                float2 u = load_u(us_t + (uint32_t)q * pu);
                if (do_norm)
                    u = __ffma2_rn(load_pair<XT>(xs_t + (uint32_t)sl * px), coef_s[q], u);
                store_pair<GT>(ALL ? drow + q * dstep : dxb + (int64_t)(r + jj * d) * grow, u);
            }
        };
        if (active && j0 - L >= ja && j0 + B - L <= jb)
            rows(std::true_type{});
        else
            rows(std::false_type{});
    };

    // ---- stages 2 and 3 of batch b (x ring batches xc of b, xp of b - 1;
    // dout ring batches gcur, gprev): new rows j0 + q, and the rows j0 - 3 + q
    // they complete; returns the lane's warp total of the dot partials (row
    // lane / 4)
    auto stage23 = [&](int b, int xc, int xp, int gcur, int gprev) {
        const int32_t j0 = js + b * B;
        const float2 *ivn = inv_s + xc * B;  // inverse RMS of the new rows
        // slots of lagged row q: q < L in the previous batch, else in this one
        const int sx_lo = xp * B + B - L, sx_hi = xc * B - L;
        const int sg_lo = gprev * B + B - L, sg_hi = gcur * B - L;
        // FAST: every new row has its dout and all its history taps, and every
        // lagged row is an output row with all its forward taps
        bool ok = true;
        if (lane < B)
            ok = (meta_s[xc * B + lane] & 0xff) == L;
        else if (lane < 2 * B)
            ok = (meta_s[(lane - B < L ? sx_lo : sx_hi) + lane - B] >> 8) == L;
        const bool full = __all_sync(kFull, ok) && active && j0 - L >= ja && j0 + B <= je &&
                          j0 + B - L <= jb;
        const uint32_t xa = xs_t + (uint32_t)(xc * B) * px, ga = gs_t + (uint32_t)(gcur * B) * pg;
        auto rows = [&](auto fast_tag) {
            constexpr bool FAST = decltype(fast_tag)::value;
            float dotv[B];
#pragma unroll
            for (int q = 0; q < B; ++q) {
                const int32_t jn = j0 + q;
                // new row: normalised x into the ring, then y and dy
                float2 xh = zero2;
                if (FAST || (active && jn < je))
                    xh = __fmul2_rn(load_pair<XT>(xa + (uint32_t)q * px), ivn[q]);
                xr[q & 3] = xh;
                float2 dyv = zero2;
                if (FAST || (active && jn < je && jn >= ja)) {
                    const int back = FAST ? L : (meta_s[xc * B + q] & 0xff);
                    float2 acc = zero2;
#pragma unroll
                    for (int k = 0; k < KT; ++k)
                        if (FAST || k <= back)
                            acc = __ffma2_rn(w[k], xr[(q - k) & 3], acc);
                    const float2 y = __ffma2_rn(sc, acc, bias);
                    const float2 g = load_pair<GT>(ga + (uint32_t)q * pg);
                    dyv = do_silu ? __fmul2_rn(g, silu_grad2(y)) : g;
                }
                dr[q & 3] = dyv;
                // lagged row jj = jn - 3: dn, weight gradients, dot partial, u
                const int32_t jj = jn - L;
                float dv = 0.f;
                if (FAST || (active && jj >= ja && jj < jb)) {
                    const int sxl = (q < L ? sx_lo : sx_hi) + q;
                    const int fwd = FAST ? L : (meta_s[sxl] >> 8);
                    const float2 xl = xr[(q - L) & 3];
                    float2 dn = zero2;
#pragma unroll
                    for (int k = 0; k < KT; ++k)
                        if (FAST || k <= fwd) {
                            dn = __ffma2_rn(w[k], dr[(q - L + k) & 3], dn);
                            dw[k] = __ffma2_rn(xl, dr[(q - L + k) & 3], dw[k]);
                        }
                    db = __fadd2_rn(db, dr[(q - L) & 3]);
                    const float2 t = __fmul2_rn(dn, xl);
                    dnw = __fadd2_rn(dnw, t);
                    const float2 st = __fmul2_rn(sc, t);
                    dv = st.x + st.y;
                    // (rows of the previous batch: their inverse RMS from its stage 2)
                    float2 u = __fmul2_rn(__fmul2_rn(sc, inv_s[sxl]), dn);
                    if (do_res)
                        u = __fadd2_rn(
                            u, load_pair<GT>(gs_t + (uint32_t)((q < L ? sg_lo : sg_hi) + q) * pg));
                    store_u(us_t + (uint32_t)q * pu, u);
                }
                dotv[q] = dv;
            }
            return warp_sum8(dotv, lane);
        };
        return full ? rows(std::true_type{}) : rows(std::false_type{});
    };

    // The batches are pipelined so that one barrier separates them: iteration
    // b finishes batch b - 1 (stage 4), computes batch b (stages 2 and 3) and
    // posts the squares of batch b + 1 (stage 1); partials are double-buffered
    // by batch parity, so a warp that runs ahead never overwrites partials
    // another warp still reads.
    stage1(0, 0);
    end_phase(0, 0, -1, 0, 0);
    if (wid == iwarp && a.ahead < nbatch)
        issue_next(a.ahead);
    // ring batches of batches b, b - 1 and b - 2 (those of batches before the
    // first are never read: their rows precede js)
    int x0 = 0, x1 = nbx - 1, x2 = nbx - 2, g0 = 0, g1 = nbg - 1;
    for (int b = 0; b < nbatch; ++b) {
        if (b > 0)
            stage4(b - 1, x1, x2);
        const float dsum = stage23(b, x0, x1, g0, g1);
        if (do_norm)
            post(dot_part + (b & 1) * PB, dsum);
        const int xn = x0 + 1 == nbx ? 0 : x0 + 1;
        if (b + 1 < nbatch)
            stage1(b + 1, xn);
        if (wid == iwarp)
            store_pending();
        end_phase(b + 1 < nbatch ? b + 1 : -1, xn * B, b, x1 * B + B - L, x0 * B - L);
        if (wid == iwarp && b + 1 + a.ahead < nbatch)
            issue_next(b + 1 + a.ahead);
        x2 = x1;
        x1 = x0;
        x0 = xn;
        g1 = g0;
        g0 = g0 + 1 == nbg ? 0 : g0 + 1;
    }
    stage4(nbatch - 1, x1, x2);

    // partials of this block: s * dw per tap, dbias, dnorm_w (zero without the norm)
    if (active) {
        auto put = [&](int q, float2 v) {
            *reinterpret_cast<float2 *>(part + (size_t)q * a.C) = v;
        };
#pragma unroll
        for (int k = 0; k < KT; ++k)
            put(k, __fmul2_rn(sc, dw[k]));
        put(KT, db);
        put(KT + 1, do_norm ? dnw : zero2);
    }
    if (timed_out && lane == 0)
        raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
    // a block leaves only once every partner has received everything it
    // stored into the partner's shared memory
    if (cs > 1)
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
