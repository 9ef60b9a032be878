// backward.cuh -- compact row gradients of the table lookup.
//
// Qwen3.8-Flash-Next engram API page, class Qwen3_8_FlashNextOwnerShardedEmbedding:
// the backward routes output gradients back to the row owner, and only the
// owner accumulates each row's gradient. With the whole table on one GPU the
// owner is this GPU, and the gradient is kept compact: the distinct rows in
// ascending order and one fp32 sum per row, never a dense table gradient.
//
// Stage 1 (sort): radix_sort.cuh orders the (row, lookup) pairs by row.
//
// Stage 2 (reduce): the sorted items are cut into one contiguous range per
// resident warp. A segment is a run of equal keys. seg_count counts segment
// heads per range and per block; seg_reduce turns those counts into each
// range's first segment index, then streams the dout rows of its range through
// a shared-memory ring filled by cp.async (several rows in flight per warp,
// independent of registers) and sums each segment in fp64 (rounded once to
// fp32 on output, so hot rows with thousands of terms stay at fp32-rounding
// distance from the exact sum). Segments that start and end inside a range are
// written directly, with each store instruction covering contiguous bytes; the
// pieces of segments that cross range boundaries are written as fp64 partial
// sums and combined, in range order, by seg_fixup (one warp per crossing
// segment). No atomics touch the sums, so the result is deterministic and hot
// rows spread over many warps.
#pragma once

#include "common.cuh"
#include "radix_sort.cuh"

namespace engram {
namespace bwd {

constexpr int kSegThreads = 256;
constexpr int kSegWarps = kSegThreads / 32;
constexpr int kSegStages = 3;      // cp.async ring depth per warp
constexpr int kSegMaxBatch = 8;    // rows per stage
constexpr int kSegStageBytes = 4096;

// ------------------------------------------------------------------ reduce

struct SegMeta {
    int32_t pe_valid; // the range's last segment has its head here and goes on
    int32_t pe_u;     // that segment's index
    int32_t pe_key;   // its row
    int32_t pb_ends;  // the segment continued into this range ends inside it
};

__device__ __forceinline__ void range_of(int64_t n, int64_t w, int64_t W, int64_t &a,
                                         int64_t &b)
{
    a = n * w / W;
    b = n * (w + 1) / W;
}

// Segment heads (first item, or key differs from the previous one) per range
// (wcount) and per block of kSegWarps ranges (bcount). The run of key
// `absent` (absent lookups; it sorts last) is not counted, so num_unique
// leaves it out; its sum lands past the counted rows.
__global__ void __launch_bounds__(kSegThreads)
    seg_count(const unsigned long long *__restrict__ items, int64_t n, int W, uint32_t absent,
              uint32_t *__restrict__ wcount, uint32_t *__restrict__ bcount)
{
    __shared__ uint32_t s_cnt[kSegWarps];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * kSegWarps + wib;
    uint32_t cnt = 0;
    if (w < W) {
        int64_t a, b;
        range_of(n, w, W, a, b);
        for (int64_t c0 = a; c0 < b; c0 += 128) {
            uint32_t key[4], prev[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t i = c0 + 32 * q + lane;
                key[q] = i < b ? item_key(__ldg(items + i)) : 0u;
                prev[q] = (i < b && i > 0) ? item_key(__ldg(items + i - 1)) : ~key[q];
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t i = c0 + 32 * q + lane;
                cnt += __popc(__ballot_sync(kFull, i < b && key[q] != prev[q] && key[q] != absent));
            }
        }
        if (lane == 0)
            wcount[w] = cnt;
    }
    if (lane == 0)
        s_cnt[wib] = w < W ? cnt : 0u;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t t = 0;
        for (int k = 0; k < kSegWarps; ++k)
            t += s_cnt[k];
        bcount[blockIdx.x] = t;
    }
}

// Four consecutive columns (float4 group f) of one staged row, as fp32.
template <int DT>
__device__ __forceinline__ float4 load_quad(const unsigned char *row, int f)
{
    if constexpr (DT == ENGRAM_F32) {
        return *(const float4 *)(row + 16 * f);
    } else if constexpr (DT == ENGRAM_BF16) {
        const uint2 v = *(const uint2 *)(row + 8 * f);
        return make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u),
                           __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
    } else {
        const uint2 v = *(const uint2 *)(row + 8 * f);
        __half2 a, b;
        memcpy(&a, &v.x, 4);
        memcpy(&b, &v.y, 4);
        const float2 fa = __half22float2(a), fb = __half22float2(b);
        return make_float4(fa.x, fa.y, fb.x, fb.y);
    }
}

// Running sum of one segment on one lane's column groups. A segment of one
// lookup is its fp32 row, copied exactly; from the second lookup on the sum
// is kept in fp64 (the first two terms added exactly) and rounded once.
template <int GF>
struct SegAcc {
    float4 first[GF];
    double acc[GF][4];
    int cnt; // lookups in the segment, saturating at 2

    __device__ __forceinline__ void add(int g, const float4 &v)
    {
        if (cnt == 0) {
            first[g] = v;
        } else if (cnt == 1) {
            acc[g][0] = (double)first[g].x + (double)v.x;
            acc[g][1] = (double)first[g].y + (double)v.y;
            acc[g][2] = (double)first[g].z + (double)v.z;
            acc[g][3] = (double)first[g].w + (double)v.w;
        } else {
            acc[g][0] += (double)v.x;
            acc[g][1] += (double)v.y;
            acc[g][2] += (double)v.z;
            acc[g][3] += (double)v.w;
        }
    }

    __device__ __forceinline__ float4 rounded(int g) const
    {
        if (cnt <= 1)
            return first[g];
        return make_float4((float)acc[g][0], (float)acc[g][1], (float)acc[g][2],
                           (float)acc[g][3]);
    }

    __device__ __forceinline__ double exact(int g, int q) const
    {
        if (cnt <= 1) {
            const float4 f = first[g];
            return (double)(q == 0 ? f.x : q == 1 ? f.y : q == 2 ? f.z : f.w);
        }
        return acc[g][q];
    }
};

// Row gradient: lane owns float4 groups f = lane + 32 g, so each store
// instruction covers contiguous bytes.
template <int GF>
__device__ __forceinline__ void store_row(float *__restrict__ dst, const SegAcc<GF> &s,
                                          int lane, int F)
{
#pragma unroll
    for (int g = 0; g < GF; ++g) {
        const int f = lane + 32 * g;
        if (f < F)
            st_stream((float4 *)dst + f, s.rounded(g));
    }
}

// Partial sum of a segment piece, kept in fp64.
template <int GF>
__device__ __forceinline__ void store_partial(double *__restrict__ dst, const SegAcc<GF> &s,
                                              int lane, int F)
{
#pragma unroll
    for (int g = 0; g < GF; ++g) {
        const int f = lane + 32 * g;
        if (f < F) {
            double2 *p = (double2 *)(dst + 4 * f);
            p[0] = make_double2(s.exact(g, 0), s.exact(g, 1));
            p[1] = make_double2(s.exact(g, 2), s.exact(g, 3));
        }
    }
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_commit()
{
    asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Segmented sums over one contiguous range of sorted items per warp.
// DT: dout dtype; GF: float4 column groups per lane (dim <= 128 * GF);
// RVT: 16-byte vectors per dout row when fixed at compile time (0: runtime).
// Dynamic shared memory: kSegWarps * kSegStages * (stage bytes + batch items).
template <int DT, int GF, int RVT>
__global__ void __launch_bounds__(kSegThreads)
    seg_reduce(const unsigned long long *__restrict__ items, int64_t n, int W,
               const uint32_t *__restrict__ wcount, const uint32_t *__restrict__ bcount,
               const void *__restrict__ dout, int dim, int batch, int stage_bytes,
               int32_t *__restrict__ uniq, float *__restrict__ grads,
               double *__restrict__ pb, double *__restrict__ pe, SegMeta *__restrict__ meta,
               int32_t *__restrict__ num_unique)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ uint32_t s_warp[32];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * kSegWarps + wib;
    const int F = dim >> 2; // float4 groups per row
    const int rvec = RVT ? RVT : dim * (DT == ENGRAM_F32 ? 4 : 2) / 16;

    // First segment index of each range: heads in earlier blocks + earlier warps.
    uint32_t before = 0;
    for (int k = threadIdx.x; k < (int)blockIdx.x; k += kSegThreads)
        before += bcount[k];
    uint32_t block_before;
    (void)block_exclusive_scan(before, s_warp, &block_before);
    uint32_t warp_before = 0;
    for (int k = 0; k < wib; ++k) {
        const int64_t wk = (int64_t)blockIdx.x * kSegWarps + k;
        warp_before += wk < W ? wcount[wk] : 0u;
    }
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0)
        *num_unique = (int32_t)(block_before + bcount[blockIdx.x]);
    if (w >= W)
        return;

    int64_t a, b;
    range_of(n, w, W, a, b);
    const int len = (int)(b - a);
    const unsigned long long *wit = items + a;
    const int stage_stride = stage_bytes + kSegMaxBatch * 8;
    unsigned char *ring = smem + (size_t)wib * kSegStages * stage_stride;
    const uint4 *drows = (const uint4 *)dout;

    // Copies of batch k (range offsets k*batch ...) into stage k % kSegStages.
    auto issue = [&](int k) {
        const int e0 = k * batch;
        if (e0 < len) {
            unsigned char *stage = ring + (k % kSegStages) * stage_stride;
            unsigned long long *smeta = (unsigned long long *)(stage + stage_bytes);
            const int rows = min(batch, len - e0);
            unsigned long long my = 0;
            if (lane < rows) {
                my = __ldg(wit + e0 + lane);
                smeta[lane] = my;
            }
            const int nvec = rows * rvec;
            // uniform trip count across the warp (the shuffle needs every lane)
            for (int v0 = 0; v0 < nvec; v0 += 32) {
                const int v = v0 + lane;
                const int r = min(v / rvec, rows - 1), c = v - r * rvec;
                const uint32_t j = (uint32_t)__shfl_sync(kFull, my, r);
                if (v < nvec)
                    cp_async16(stage + 16 * v, drows + (size_t)j * rvec + c);
            }
        }
        cp_async_commit();
    };

    SegAcc<GF> sa;
    sa.cnt = 0;
    int32_t u = (int32_t)(block_before + warp_before) - 1; // open segment's index
    uint32_t cur_key = 0;
    uint32_t prev_key = a > 0 ? item_key(__ldg(items + a - 1)) : ~item_key(__ldg(items + a));
    bool open_here = false; // the open segment's head lies in this range
    bool started = false;   // some lookup of this range has been added
    int32_t pb_ends = 0;

    const int nb = (len + batch - 1) / batch;
#pragma unroll
    for (int k = 0; k < kSegStages; ++k)
        issue(k);
    for (int k = 0; k < nb; ++k) {
        cp_async_wait<kSegStages - 1>();
        __syncwarp();
        const unsigned char *stage = ring + (k % kSegStages) * stage_stride;
        const unsigned long long *smeta = (const unsigned long long *)(stage + stage_bytes);
        const int rows = min(batch, len - k * batch);

        // Close the open segment (it ends just before the current row).
        auto close = [&]() {
            if (open_here) {
                store_row<GF>(grads + (size_t)u * dim, sa, lane, F);
                if (lane == 0)
                    uniq[u] = (int32_t)cur_key;
            } else {
                store_partial<GF>(pb + (size_t)w * dim, sa, lane, F);
                pb_ends = 1;
            }
        };

        bool all_heads = false;
        if constexpr (RVT != 0) {
            // Fast path: every row of a full batch starts its own segment (the
            // common case when rows are nearly all distinct). Rows 0..rows-2
            // are then complete one-lookup segments whose gradients are the
            // rows themselves, and their outputs are contiguous in grads:
            // convert and copy with fully coalesced stores.
            const uint32_t mykey = lane < rows ? item_key(smeta[lane]) : 0u;
            uint32_t up = __shfl_up_sync(kFull, mykey, 1);
            if (lane == 0)
                up = prev_key;
            const uint32_t repeats = __ballot_sync(kFull, lane < rows && mykey == up);
            all_heads = rows == batch && repeats == 0;
            if (all_heads) {
                if (started)
                    close();
                constexpr int FT = RVT * 16 / (DT == ENGRAM_F32 ? 16 : 8); // float4 groups per row
                const int32_t ub = u + 1; // segment index of row 0
                const int nv = (rows - 1) * FT;
                float4 *gdst = (float4 *)(grads + (size_t)ub * dim);
                for (int v = lane; v < nv; v += 32) {
                    const int r = v / FT, f = v - r * FT;
                    st_stream(gdst + v, load_quad<DT>(stage + r * RVT * 16, f));
                }
                if (lane < rows - 1)
                    uniq[ub + lane] = (int32_t)mykey;
                // the last row opens the next segment
                const int rl = rows - 1;
                sa.cnt = 0;
#pragma unroll
                for (int g = 0; g < GF; ++g) {
                    const int f = lane + 32 * g;
                    if (f < F)
                        sa.add(g, load_quad<DT>(stage + rl * RVT * 16, f));
                }
                sa.cnt = 1;
                u = ub + rl;
                cur_key = __shfl_sync(kFull, mykey, rl);
                prev_key = cur_key;
                open_here = true;
                started = true;
            }
        }
        if (!all_heads) {
            for (int r = 0; r < rows; ++r) {
                const uint32_t key = item_key(smeta[r]);
                if (key != prev_key) {
                    if (started)
                        close();
                    ++u;
                    cur_key = key;
                    open_here = true;
                    sa.cnt = 0;
                }
                prev_key = key;
                started = true;
                const unsigned char *row = stage + r * rvec * 16;
#pragma unroll
                for (int g = 0; g < GF; ++g) {
                    const int f = lane + 32 * g;
                    if (f < F)
                        sa.add(g, load_quad<DT>(row, f));
                }
                sa.cnt = min(sa.cnt + 1, 2);
            }
        }
        __syncwarp();
        issue(k + kSegStages);
    }
    cp_async_wait<0>();

    // The range's last segment: does it go on past b?
    const bool cont = b < n && item_key(__ldg(items + b)) == prev_key;
    int32_t pe_valid = 0;
    if (open_here) {
        if (cont) {
            store_partial<GF>(pe + (size_t)w * dim, sa, lane, F);
            pe_valid = 1;
        } else {
            store_row<GF>(grads + (size_t)u * dim, sa, lane, F);
            if (lane == 0)
                uniq[u] = (int32_t)cur_key;
        }
    } else {
        // no head in the range: it is one piece of a segment begun earlier
        store_partial<GF>(pb + (size_t)w * dim, sa, lane, F);
        pb_ends = cont ? 0 : 1;
    }
    if (lane == 0)
        meta[w] = SegMeta{pe_valid, u, (int32_t)cur_key, pb_ends};
}

// One warp per segment that crosses range boundaries: its head piece plus the
// following ranges' pieces, in range order.
template <int GF>
__global__ void __launch_bounds__(kSegThreads)
    seg_fixup(int W, int dim, const double *__restrict__ pb, const double *__restrict__ pe,
              const SegMeta *__restrict__ meta, int32_t *__restrict__ uniq,
              float *__restrict__ grads)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= W)
        return;
    const SegMeta m = meta[w];
    if (!m.pe_valid)
        return;
    const int F = dim >> 2;
    double acc[GF][4];
#pragma unroll
    for (int g = 0; g < GF; ++g) {
        const int f = lane + 32 * g;
#pragma unroll
        for (int q = 0; q < 4; ++q)
            acc[g][q] = f < F ? pe[(size_t)w * dim + 4 * f + q] : 0.0;
    }
    for (int64_t w2 = w + 1; w2 < W; ++w2) {
#pragma unroll
        for (int g = 0; g < GF; ++g) {
            const int f = lane + 32 * g;
            if (f < F) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    acc[g][q] += pb[(size_t)w2 * dim + 4 * f + q];
            }
        }
        if (meta[w2].pb_ends)
            break;
    }
#pragma unroll
    for (int g = 0; g < GF; ++g) {
        const int f = lane + 32 * g;
        if (f < F)
            st_stream((float4 *)(grads + (size_t)m.pe_u * dim) + f,
                      make_float4((float)acc[g][0], (float)acc[g][1], (float)acc[g][2],
                                  (float)acc[g][3]));
    }
    if (lane == 0)
        uniq[m.pe_u] = m.pe_key;
}

} // namespace bwd
} // namespace engram
