// ple_conv_reg.cuh -- the PLE tail of ple_conv.cuh for a kernel width KT and
// dilation DT fixed at compile time (the page's 4 and 3), with the
// convolution's history held in registers instead of shared memory.
//
// Taps of row t read rows t - DT, ..., t - (KT-1)*DT, all of t's residue
// modulo DT. A thread therefore keeps, for each residue, the last KT-1
// normalised values of its 8 channels in registers; walking rows in blocks of
// DT*(KT-1) (the halo, 9 on the page) makes every register index static:
// row j of a block (group q = j / DT, residue j % DT) reads history slot
// (q - k) mod (KT-1) for tap k and then overwrites slot q.
//
// Rows travel a block at a time through a ring of up to four shared-memory
// buffers, and the block is warp-specialised:
//   - two RMS warps: one of them moves each chunk's rows into a buffer with
//     cp.async.bulk (completion on the buffer's mbarrier, waited on with a
//     time bound) and sends the following chunk towards L2; both compute each
//     row's inverse RMS from shared memory (one warp per row) and the rows'
//     counts of in-sequence history taps, and mark the blocks whose rows all
//     have full history and an output;
//   - conv warps (the others): thread v owns 8 channels of the branch (G / 8
//     threads), reads them from the buffer, and normalises, convolves,
//     applies SiLU and the residual, storing straight to global memory.
// Hand-over per buffer b uses three mbarriers: the bulk copies complete
// "landed"; each RMS warp arrives on "described" when its rows, counts and
// flags are written; each conv warp waits on "described" on its own (conv
// warps drift apart by up to the ring depth, never waiting for one another)
// and arrives on "consumed" when done; the loading warp waits on "consumed"
// before reusing the buffer. Every wait is bounded in time: one that runs out
// raises ENGRAM_DEVERR_COPY_TIMEOUT and the thread skips its later waits on
// the other warps (not those on its own bulk copies), so the kernel always
// ends promptly, on stale data.
#pragma once

#include "ple_conv.cuh"

namespace engram {
namespace ple {

constexpr int kRegRmsWarps = 2;
constexpr int kRegMaxConvWarps = 10;  // 8 channels per thread: G <= 2560
constexpr int kRegThreads = 32 * (kRegMaxConvWarps + kRegRmsWarps);
constexpr int kRegMaxBufs = 4;        // row buffers, at most (one block each)
constexpr int kRegMaxBlockRows = 9;   // rows per block, at most
constexpr uint64_t kCopyWaitNs = 500ull * 1000 * 1000;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

// One contiguous global -> shared copy by the bulk-copy (TMA) engine,
// completing `bytes` of transaction count on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Waits (bounded by kCopyWaitNs) for phase `parity` of `bar`; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t addr = smem_u32(bar);
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
        uint64_t now;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
        if (spin == 0)
            t0 = now;
        else if (now - t0 > kCopyWaitNs)
            return false;
    }
}

// Shared memory: inverse RMS [4][9] float, tap counts [4][9] int32,
// full-block flags [4] int32, and per buffer three mbarriers (rows landed,
// rows described, rows consumed); then the row buffers [bufs][9][pitch].
constexpr int kRegOffNv = kRegMaxBufs * kRegMaxBlockRows * 4;
constexpr int kRegOffFast = 2 * kRegOffNv;
constexpr int kRegOffBars = kRegOffFast + kRegMaxBufs * 4;
constexpr int kRegHeader = kRegOffBars + 3 * kRegMaxBufs * 8;
constexpr int kRegDataOffset = (kRegHeader + 127) / 128 * 128;

__host__ __device__ constexpr size_t reg_smem_bytes(int bufs, int block_rows, int pitch)
{
    return (size_t)kRegDataOffset + (size_t)bufs * block_rows * pitch;
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

template <typename XT, typename OT, int KT, int DT>
__global__ void __launch_bounds__(kRegThreads, 1) short_conv_reg_kernel(const ConvArgs a)
{
    constexpr int H = KT - 1;                       // history depth per residue
    constexpr int BLK = DT * H;                     // rows per unrolled block (= halo)
    constexpr int CH = 8, NP = CH / 2;
    constexpr int EV = 16 / (int)sizeof(XT);        // channels per 16-byte vector
    constexpr int NV = CH / EV;                     // vectors per thread and row (1 or 2)
    constexpr int OB = EV * (int)sizeof(OT);        // output bytes per vector's channels
    static_assert(H >= 1, "the register path needs at least one history tap");
    static_assert(BLK <= kRegMaxBlockRows, "block arrays too small");
    extern __shared__ __align__(128) unsigned char smem[];
    float *inv_s = reinterpret_cast<float *>(smem);                        // [4][9]
    int32_t *nv_s = reinterpret_cast<int32_t *>(smem + kRegOffNv);        // [4][9]
    int32_t *fast_s = reinterpret_cast<int32_t *>(smem + kRegOffFast);    // [4]
    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(smem + kRegOffBars); // [4] rows landed
    uint64_t *full_bar = tma_bar + kRegMaxBufs;                           // [4] rows described
    uint64_t *empty_bar = full_bar + kRegMaxBufs;                         // [4] rows consumed
    unsigned char *data = smem + kRegDataOffset;

    if (a.cu != nullptr)
        check_cu_seqlens(a.cu, a.nseq, a.T);

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int NT = blockDim.x;
    const int ncw = (NT >> 5) - kRegRmsWarps;  // conv warps
    const int m = blockIdx.x / a.bpg, j = blockIdx.x - m * a.bpg;
    const int64_t ta = a.T * j / a.bpg, tb = a.T * (j + 1) / a.bpg;
    if (ta >= tb)
        return;
    const int NB = a.reg_bufs;                  // row buffers, one block of BLK rows each
    const int64_t tlo = ta - BLK > 0 ? ta - BLK : 0;
    const int nblocks = (int)((tb - tlo + BLK - 1) / BLK);
    const uint32_t row_bytes = (uint32_t)a.G * sizeof(XT);
    const int pitch = a.pitch;
    const char *xbranch = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT);

    if (tid == 0) {
        for (int b = 0; b < NB; ++b) {
            mbar_init(tma_bar + b, 1);
            mbar_init(full_bar + b, kRegRmsWarps);
            mbar_init(empty_bar + b, ncw);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    bool timed_out = false;

    if (wid >= ncw) {
        // ================================================== RMS warps
        const int rw = wid - ncw;
        const int nvec = (int)(row_bytes / 16);
        const bool do_norm = a.flags & ENGRAM_CONV_NORM;
        // warp 0 of the pair moves block c's rows into buffer c % NB and sends
        // the block after it towards L2
        auto load_block = [&](int c) {
            const int64_t c0 = tlo + (int64_t)c * BLK;
            const int rc = (int)min64(BLK, tb - c0);
            const int b = c % NB;
            if (lane == 0)
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                                 smem_u32(tma_bar + b)),
                             "r"((uint32_t)rc * row_bytes)
                             : "memory");
            __syncwarp();
            if (lane < rc)
                bulk_load(data + (size_t)(b * BLK + lane) * pitch, xbranch + (c0 + lane) * xrow,
                          row_bytes, tma_bar + b);
            const int64_t n0 = c0 + BLK;
            if (lane < BLK && n0 + lane < tb)
                prefetch_l2(xbranch + (n0 + lane) * xrow, row_bytes);
        };
        if (rw == 0)
            for (int c = 0; c < NB && c < nblocks; ++c)
                load_block(c);
        for (int c = 0; c < nblocks; ++c) {
            const int b = c % NB;
            const int64_t c0 = tlo + (int64_t)c * BLK;
            const int rc = (int)min64(BLK, tb - c0);
            if (!mbar_wait(tma_bar + b, (uint32_t)(c / NB) & 1u))
                timed_out = true;
            const unsigned char *buf = data + (size_t)b * BLK * pitch;
            for (int r = rw; r < rc; r += kRegRmsWarps) {
                // EV / 2 independent accumulators keep the FMA chain short
                float2 ss[EV / 2];
#pragma unroll
                for (int e = 0; e < EV / 2; ++e)
                    ss[e] = make_float2(0.f, 0.f);
#pragma unroll 2
                for (int v = lane; v < nvec; v += 32) {
                    const uint4 q = *reinterpret_cast<const uint4 *>(buf + (size_t)r * pitch +
                                                                     (size_t)v * 16);
                    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
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
                if (lane == 0)
                    inv_s[b * kRegMaxBlockRows + r] =
                        do_norm ? rsqrtf(fmaf(tot, a.inv_G, a.eps)) : 1.f;
            }
            if (rw == 1) {
                int nv = 0;
                if (lane < rc) {
                    const int64_t t = c0 + lane;
                    const int64_t start =
                        a.cu != nullptr ? (int64_t)__ldg(a.cu + find_sequence(a.cu, a.nseq, t)) : 0;
                    const int64_t back = t - start;
                    nv = back >= BLK ? H : back <= 0 ? 0 : (int)back / DT;
                    nv_s[b * kRegMaxBlockRows + lane] = nv;
                }
                const bool row_full = lane >= BLK || (lane < rc && c0 + lane >= ta && nv == H);
                const bool full = __all_sync(kFull, row_full);
                if (lane == 0)
                    fast_s[b] = full;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(full_bar + b);  // this warp's part of block c is described
            // the buffer of block c - 1 takes block c - 1 + NB once every conv
            // warp is done with it (they worked on it while block c was being
            // described)
            if (rw == 0 && c >= 1 && c - 1 + NB < nblocks) {
                const int pb = (c - 1) % NB;
                if (!timed_out && !mbar_wait(empty_bar + pb, (uint32_t)((c - 1) / NB) & 1u))
                    timed_out = true;
                load_block(c - 1 + NB);
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
    float2 wk[KT][NP];
    float2 bias[NP];
#pragma unroll
    for (int e = 0; e < CH; ++e) {
        const int64_t c = (int64_t)m * a.G + (int64_t)(tid + (e / EV) * a.nth) * EV + e % EV;
        const float scale =
            active && do_norm && a.norm_w ? 1.f + load_weight(a.norm_w, a.wdtype, c) : 1.f;
        const float bv = active && a.bias ? load_weight(a.bias, a.wdtype, c) : 0.f;
        if (e & 1)
            bias[e / 2].y = bv;
        else
            bias[e / 2].x = bv;
#pragma unroll
        for (int k = 0; k < KT; ++k) {
            const float w = active ? load_weight(a.conv_w, a.wdtype, c * KT + (KT - 1 - k)) * scale
                                   : 0.f;
            if (e & 1)
                wk[k][e / 2].y = w;
            else
                wk[k][e / 2].x = w;
        }
    }
    float2 hist[DT][H][NP];
#pragma unroll
    for (int r = 0; r < DT; ++r)
#pragma unroll
        for (int s = 0; s < H; ++s)
#pragma unroll
            for (int p = 0; p < NP; ++p)
                hist[r][s][p] = make_float2(0.f, 0.f);

    char *out = static_cast<char *>(a.out);
    for (int c = 0; c < nblocks; ++c) {
        const int b = c % NB;
        const int64_t c0 = tlo + (int64_t)c * BLK;
        const int rc = (int)min64(BLK, tb - c0);
        // block c described (after a timeout, later waits are skipped so the
        // kernel ends promptly)
        if (!timed_out && !mbar_wait(full_bar + b, (uint32_t)(c / NB) & 1u))
            timed_out = true;
        const unsigned char *mine = data + (size_t)b * BLK * pitch + (size_t)tid * 16;
        // FAST: every row of the block has its full history and an output
        auto run_block = [&](auto fast_tag) {
            constexpr bool FAST = decltype(fast_tag)::value;
#pragma unroll
            for (int jj = 0; jj < BLK; ++jj) {
                const int q = jj / DT, res = jj % DT;
                const int64_t t = c0 + jj;
                const bool valid = FAST || jj < rc;
                float xv[CH];
#pragma unroll
                for (int v = 0; v < NV; ++v) {
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    if (active && valid) {
                        const uint4 u4 = *reinterpret_cast<const uint4 *>(
                            mine + (size_t)jj * pitch + (size_t)v * a.nth * 16);
                        w[0] = u4.x;
                        w[1] = u4.y;
                        w[2] = u4.z;
                        w[3] = u4.w;
                    }
                    Elem<XT>::template unpack<EV>(w, &xv[v * EV]);
                }
                const float inv = valid ? inv_s[b * kRegMaxBlockRows + jj] : 0.f;
                const float2 inv2 = make_float2(inv, inv);
                float2 n[NP], y[NP], z[NP];
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    n[p] = __fmul2_rn(make_float2(xv[2 * p], xv[2 * p + 1]), inv2);
                    y[p] = __ffma2_rn(wk[0][p], n[p], bias[p]);
                    z[p] = make_float2(0.f, 0.f);
                }
                int nv = H;
                if constexpr (!FAST)
                    nv = valid ? nv_s[b * kRegMaxBlockRows + jj] : 0;
                // taps in two chains (odd into z) to halve the dependent length
#pragma unroll
                for (int k = 1; k <= H; ++k) {
                    const int s = (q - k + H * DT) % H;  // static slot of row t - k * DT
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        float2 h = hist[res][s][p];
                        if constexpr (!FAST)
                            h = k <= nv ? h : make_float2(0.f, 0.f);
                        if (k & 1)
                            z[p] = __ffma2_rn(wk[k][p], h, z[p]);
                        else
                            y[p] = __ffma2_rn(wk[k][p], h, y[p]);
                    }
                }
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    y[p] = __fadd2_rn(y[p], z[p]);
                    hist[res][q % H][p] = n[p];
                }
                if (do_silu) {
#pragma unroll
                    for (int p = 0; p < NP; ++p)
                        y[p] = silu2(y[p]);
                }
                if (do_res) {
#pragma unroll
                    for (int p = 0; p < NP; ++p)
                        y[p] = __fadd2_rn(y[p], make_float2(xv[2 * p], xv[2 * p + 1]));
                }
                if (active && (FAST || (valid && t >= ta))) {
                    const int64_t off = t * a.C + (int64_t)m * a.G;
                    float o[CH];
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        o[2 * p] = y[p].x;
                        o[2 * p + 1] = y[p].y;
                    }
#pragma unroll
                    for (int v = 0; v < NV; ++v) {
                        uint32_t w[OB / 4];
                        Elem<OT>::template pack<EV>(&o[v * EV], w);
                        store_words<OB>(
                            out + (off + (int64_t)(tid + v * a.nth) * EV) * sizeof(OT), w);
                    }
                }
            }
        };
        if (fast_s[b])
            run_block(std::true_type{});
        else
            run_block(std::false_type{});
        __syncwarp();
        if (lane == 0)
            mbar_arrive(empty_bar + b);  // this warp is done with buffer b
    }
    if (timed_out && lane == 0)
        raise_device_error(ENGRAM_DEVERR_COPY_TIMEOUT);
}

} // namespace ple
} // namespace engram
