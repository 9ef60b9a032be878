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
// Stage 2 (reduce, one launch): the sorted items are cut into one contiguous
// range per resident warp. A segment is a run of equal keys. Each warp counts
// the segment heads in its range, publishes the count and looks back over the
// earlier warps' published counts for its first segment index (a decoupled
// look-back: a warp's count is out as soon as it is taken, and a warp that has
// its total publishes that too, so later warps stop there). Meanwhile its
// first dout rows are already on their way: the warp streams its rows through
// a shared-memory ring filled by cp.async (several rows in flight per warp,
// independent of registers) and sums each segment in fp64 (rounded once to
// fp32 on output, so hot rows with thousands of terms stay at fp32-rounding
// distance from the exact sum). Segments that start and end inside a range are
// written directly, with each store instruction covering contiguous bytes; the
// pieces of segments that cross range boundaries are written as fp64 partial
// sums, and the warp holding a crossing segment's last piece adds the pieces
// in range order once their owners have published them. No atomics touch the
// sums, so the result is deterministic and hot rows spread over many warps.
// Published words carry the launch's generation (advanced by the last warp of
// each launch), so nothing has to be cleared between launches; the sort clears
// them once. Every wait is bounded: one that runs out raises
// ENGRAM_DEVERR_REDUCE_TIMEOUT and the warp skips the writes it cannot place.
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

// Look-back state of a reduce launch, in the workspace (cleared by the sort).
struct SegSync {
    unsigned long long *status; // [W]: per warp, tag << 32 | count (tag: generation, kind)
    unsigned *ready;            // [W]: generation + 1 once the warp's partials are out
    unsigned *gen;              // launch generation, advanced by each launch's last warp
    unsigned *done;             // warps of the launch that have finished
};

constexpr uint32_t kSegSpin = 1u << 22; // polls (~64 ns apart) before a wait gives up

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Segment heads (first item, or key differs from the previous one) in [a, b).
__device__ __forceinline__ uint32_t count_heads(const unsigned long long *__restrict__ items,
                                                int64_t a, int64_t b, int lane)
{
    uint32_t cnt = 0;
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
            cnt += __popc(__ballot_sync(kFull, i < b && key[q] != prev[q]));
        }
    }
    return cnt;
}

// Decoupled look-back: publishes warp w's head count `cnt` and returns the
// number of heads before its range (false if a wait ran out). Tag of a word:
// 2 * (generation + 1) + (1 if the value is the inclusive total up to that warp).
__device__ __forceinline__ bool seg_lookback(const SegSync &sy, uint32_t G, int64_t w,
                                             uint32_t cnt, int lane, uint32_t &excl)
{
    const uint32_t tag = 2u * (G + 1u);
    if (lane == 0)
        st_relaxed_u64(sy.status + w, ((unsigned long long)tag << 32) | cnt);
    excl = 0;
    int64_t base = w - 1;
    uint32_t spins = 0;
    while (base >= 0) {
        const int64_t q = base - lane;
        unsigned long long word = 0;
        bool ok = false;
        for (;;) {
            if (q >= 0) {
                word = ld_relaxed_u64(sy.status + q);
                ok = (uint32_t)(word >> 33) == G + 1u;
            } else {
                word = ((unsigned long long)(tag | 1u) << 32); // before warp 0: total 0
                ok = true;
            }
            if (__all_sync(kFull, ok))
                break;
            if (++spins > kSegSpin)
                return false;
            __nanosleep(64);
        }
        const uint32_t incl = __ballot_sync(kFull, (word >> 32) & 1u);
        const uint32_t v = (uint32_t)word;
        if (incl) {
            const int k = __ffs(incl) - 1; // the nearest inclusive total
            excl += __reduce_add_sync(kFull, lane <= k ? v : 0u);
            break;
        }
        excl += __reduce_add_sync(kFull, v);
        base -= 32;
    }
    if (lane == 0)
        st_relaxed_u64(sy.status + w, ((unsigned long long)(tag | 1u) << 32) | (excl + cnt));
    return true;
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
    seg_reduce(const unsigned long long *__restrict__ items, int64_t n, int W, SegSync sy,
               const void *__restrict__ dout, int dim, int batch, int stage_bytes,
               int32_t *__restrict__ uniq, float *__restrict__ grads,
               double *__restrict__ pb, double *__restrict__ pe, SegMeta *__restrict__ meta,
               int32_t *__restrict__ num_unique)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int64_t w = (int64_t)blockIdx.x * kSegWarps + wib;
    const int F = dim >> 2; // float4 groups per row
    const int rvec = RVT ? RVT : dim * (DT == ENGRAM_F32 ? 4 : 2) / 16;
    if (w >= W)
        return;
    const uint32_t G = *(volatile const unsigned *)sy.gen; // set before this launch

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

#pragma unroll
    for (int k = 0; k < kSegStages; ++k)
        issue(k);

    // First segment index of the range, while the first rows are in flight.
    const uint32_t cnt = count_heads(items, a, b, lane);
    uint32_t excl = 0;
    const bool placed = seg_lookback(sy, G, w, cnt, lane, excl);
    if (w == W - 1 && lane == 0 && placed)
        *num_unique = (int32_t)(excl + cnt);
    if (!placed) {
        if (lane == 0)
            raise_device_error(ENGRAM_DEVERR_REDUCE_TIMEOUT);
        cp_async_wait<0>();
        // nothing of this range can be placed; let the launch finish
        if (lane == 0) {
            __threadfence();
            *(volatile unsigned *)(sy.ready + w) = G + 1u;
            if (atomicAdd(sy.done, 1u) == (unsigned)W - 1u) {
                *(volatile unsigned *)sy.done = 0u;
                __threadfence();
                atomicAdd(sy.gen, 1u);
            }
        }
        return;
    }
    const uint32_t first_key = item_key(__ldg(items + a));

    SegAcc<GF> sa;
    sa.cnt = 0;
    int32_t u = (int32_t)excl - 1; // open segment's index
    uint32_t cur_key = 0;
    uint32_t prev_key = a > 0 ? item_key(__ldg(items + a - 1)) : ~item_key(__ldg(items + a));
    bool open_here = false; // the open segment's head lies in this range
    bool started = false;   // some lookup of this range has been added
    int32_t pb_ends = 0;

    const int nb = (len + batch - 1) / batch;
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
    if (lane == 0) {
        meta[w] = SegMeta{pe_valid, u, (int32_t)cur_key, pb_ends};
        __threadfence();
        *(volatile unsigned *)(sy.ready + w) = G + 1u; // this range's pieces are out
    }
    __syncwarp();

    // The range holds the last piece of a segment begun in an earlier range:
    // find the range with its head piece (pe) and add the pieces in range
    // order -- head piece, the earlier ranges' pieces, this range's (pb).
    if (pb_ends) {
        int64_t wh = -1;
        uint32_t spins = 0;
        for (int64_t base = w - 1; wh < 0 && base >= 0; base -= 32) {
            const int64_t q = base - lane;
            bool ok = q < 0;
            while (!__all_sync(kFull, ok)) {
                if (!ok)
                    ok = *(volatile const unsigned *)(sy.ready + q) == G + 1u;
                if (++spins > kSegSpin)
                    break;
                __nanosleep(64);
            }
            if (!__all_sync(kFull, ok)) {
                wh = -2;
                break;
            }
            __threadfence();
            const bool head = q >= 0 && __ldcg(&meta[q].pe_valid) != 0;
            const uint32_t hm = __ballot_sync(kFull, head);
            if (hm)
                wh = base - (__ffs(hm) - 1);
        }
        if (wh < 0) {
            if (lane == 0)
                raise_device_error(ENGRAM_DEVERR_REDUCE_TIMEOUT);
        } else {
            double acc[GF][4];
#pragma unroll
            for (int g = 0; g < GF; ++g) {
                const int f = lane + 32 * g;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    acc[g][q] = f < F ? __ldcg(pe + (size_t)wh * dim + 4 * f + q) : 0.0;
            }
            for (int64_t w2 = wh + 1; w2 <= w; ++w2) {
#pragma unroll
                for (int g = 0; g < GF; ++g) {
                    const int f = lane + 32 * g;
                    if (f < F) {
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            acc[g][q] += __ldcg(pb + (size_t)w2 * dim + 4 * f + q);
                    }
                }
            }
            const int32_t uc = (int32_t)excl - 1; // the segment continued into this range
#pragma unroll
            for (int g = 0; g < GF; ++g) {
                const int f = lane + 32 * g;
                if (f < F)
                    st_stream((float4 *)(grads + (size_t)uc * dim) + f,
                              make_float4((float)acc[g][0], (float)acc[g][1], (float)acc[g][2],
                                          (float)acc[g][3]));
            }
            if (lane == 0)
                uniq[uc] = (int32_t)first_key;
        }
    }

    // The launch's last warp advances the generation for the next launch.
    if (lane == 0) {
        __threadfence();
        if (atomicAdd(sy.done, 1u) == (unsigned)W - 1u) {
            *(volatile unsigned *)sy.done = 0u;
            __threadfence();
            atomicAdd(sy.gen, 1u);
        }
    }
}

} // namespace bwd
} // namespace engram
