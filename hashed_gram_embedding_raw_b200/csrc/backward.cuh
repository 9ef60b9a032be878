// backward.cuh -- compact row gradients of the table lookup.
//
// Qwen3.8-Flash-Next engram API page, class Qwen3_8_FlashNextOwnerShardedEmbedding:
// the backward routes output gradients back to the row owner, and only the
// owner accumulates each row's gradient. With the whole table on one GPU the
// owner is this GPU, and the gradient is kept compact: the distinct rows in
// ascending order and one fp32 sum per row, never a dense table gradient.
//
// Stage 1 (sort): the pairs (idx[j], j) are packed as 64-bit items
// key << 32 | j and sorted by key with a stable least-significant-digit radix
// sort, 8 bits per pass, ceil(bits(table_rows - 1) / 8) passes. Each pass is
// reduce-then-scan: per-tile digit counts (upsweep), an exclusive scan of the
// counts of each digit over tiles (scan), and a stable in-tile ranking with
// warp match/ballot, staged through shared memory so the scatter writes
// contiguous runs (downsweep). No block ever waits on another block.
//
// Stage 2 (reduce): the sorted items are cut into one contiguous range per
// warp. A segment is a run of equal keys. Warps count segment heads in their
// ranges, a single-block scan turns the counts into each range's first
// segment index, and each warp then sums dout rows along its range in fp64
// (rounded once to fp32 on output, so hot rows with thousands of terms stay
// within a few fp32 ulps of the exact sum):
// segments that start and end inside the range are written directly; the
// pieces of segments that cross range boundaries are written as partial sums
// and combined, in range order, by one warp per crossing segment. Hot rows
// (thousands of lookups of one row) are thereby spread over many warps with
// no atomics, and the result is deterministic.
#pragma once

#include "common.cuh"

namespace engram {
namespace bwd {

constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems; // 4096 pairs per tile
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;
constexpr int kSortWarps = kSortThreads / 32;
static_assert(kRadix == kSortThreads, "one thread per digit");

constexpr int kSegThreads = 256;
constexpr int kSegPrefetch = 8; // dout rows in flight per warp

__device__ __forceinline__ uint32_t item_key(uint64_t it) { return (uint32_t)(it >> 32); }

// Pass 0 reads the int32 indices and forms the items; later passes read items.
template <bool FIRST>
__device__ __forceinline__ uint64_t load_item(const void *__restrict__ src, int64_t i)
{
    if constexpr (FIRST) {
        const uint32_t key = (uint32_t)__ldg((const int32_t *)src + i);
        return ((uint64_t)key << 32) | (uint32_t)i;
    } else {
        return __ldg((const unsigned long long *)src + i);
    }
}

// Per-tile digit counts, stored digit-major: hist[d * ntiles + tile].
template <bool FIRST>
__global__ void __launch_bounds__(kSortThreads)
    radix_upsweep(const void *__restrict__ src, int64_t n, int shift, uint32_t rows,
                  uint32_t *__restrict__ hist, int ntiles)
{
    __shared__ uint32_t s_cnt[kRadix];
    s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    bool bad = false;
#pragma unroll 4
    for (int r = 0; r < kSortItems; ++r) {
        const int64_t i = base + (int64_t)r * kSortThreads + threadIdx.x;
        const bool valid = i < n;
        uint32_t d = kRadix; // sentinel shared by the lanes past the end
        if (valid) {
            const uint32_t key = item_key(load_item<FIRST>(src, i));
            if (FIRST && key >= rows)
                bad = true;
            d = (key >> shift) & (kRadix - 1);
        }
        const uint32_t peers = __match_any_sync(kFull, d);
        if (valid && lane == __ffs(peers) - 1)
            atomicAdd(&s_cnt[d], (uint32_t)__popc(peers));
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    __syncthreads();
    hist[(size_t)threadIdx.x * ntiles + blockIdx.x] = s_cnt[threadIdx.x];
}

// One block per digit: exclusive scan of that digit's counts over the tiles
// (in place) and the digit's total.
__global__ void __launch_bounds__(kSortThreads)
    radix_scan(uint32_t *__restrict__ hist, int ntiles, uint32_t *__restrict__ totals)
{
    __shared__ uint32_t s_warp[32];
    uint32_t *row = hist + (size_t)blockIdx.x * ntiles;
    uint32_t carry = 0;
    for (int t0 = 0; t0 < ntiles; t0 += kSortThreads * 4) {
        uint32_t v[4], sum = 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int t = t0 + threadIdx.x * 4 + q;
            v[q] = t < ntiles ? row[t] : 0u;
            sum += v[q];
        }
        uint32_t tot;
        uint32_t run = carry + block_exclusive_scan(sum, s_warp, &tot);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int t = t0 + threadIdx.x * 4 + q;
            if (t < ntiles)
                row[t] = run;
            run += v[q];
        }
        carry += tot;
    }
    if (threadIdx.x == 0)
        totals[blockIdx.x] = carry;
}

// Stable scatter of one tile to its sorted positions.
template <bool FIRST>
__global__ void __launch_bounds__(kSortThreads)
    radix_downsweep(const void *__restrict__ src, unsigned long long *__restrict__ dst,
                    int64_t n, int shift, const uint32_t *__restrict__ hist,
                    const uint32_t *__restrict__ totals, int ntiles)
{
    __shared__ uint32_t s_whist[kSortWarps][kRadix];
    __shared__ uint32_t s_tstart[kRadix];
    __shared__ uint32_t s_gbase[kRadix];
    __shared__ uint32_t s_warp[32];
    __shared__ unsigned long long s_items[kSortTile];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int k = tid; k < kSortWarps * kRadix; k += kSortThreads)
        (&s_whist[0][0])[k] = 0;
    __syncthreads();

    // Each warp ranks its own 32 * kSortItems consecutive items, in order.
    const int64_t base = (int64_t)blockIdx.x * kSortTile;
    const int64_t wbase = base + (int64_t)wid * (32 * kSortItems);
    const uint32_t lt = lanemask_lt();
    uint64_t it[kSortItems];
    uint32_t rank[kSortItems];
#pragma unroll
    for (int r = 0; r < kSortItems; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        const bool valid = i < n;
        it[r] = valid ? load_item<FIRST>(src, i) : 0ull;
        const uint32_t d = valid ? (item_key(it[r]) >> shift) & (kRadix - 1) : kRadix;
        const uint32_t peers = __match_any_sync(kFull, d);
        const int leader = __ffs(peers) - 1;
        uint32_t cnt = 0;
        if (valid && lane == leader) {
            cnt = s_whist[wid][d];
            s_whist[wid][d] = cnt + __popc(peers);
        }
        cnt = __shfl_sync(kFull, cnt, leader);
        rank[r] = cnt + __popc(peers & lt);
        __syncwarp();
    }
    __syncthreads();

    // Thread d: offsets of digit d for every warp (in warp order), the
    // digit's start inside the tile, and its global base.
    uint32_t tcount = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
        const uint32_t c = s_whist[w][tid];
        s_whist[w][tid] = tcount;
        tcount += c;
    }
    const uint32_t tstart = block_exclusive_scan(tcount, s_warp, nullptr);
    const uint32_t dbase = block_exclusive_scan(totals[tid], s_warp, nullptr);
    s_tstart[tid] = tstart;
    s_gbase[tid] = dbase + hist[(size_t)tid * ntiles + blockIdx.x] - tstart;
    __syncthreads();

#pragma unroll
    for (int r = 0; r < kSortItems; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < n) {
            const uint32_t d = (item_key(it[r]) >> shift) & (kRadix - 1);
            s_items[s_tstart[d] + s_whist[wid][d] + rank[r]] = it[r];
        }
    }
    __syncthreads();
    const int tile_n = (int)min64(kSortTile, n - base);
    for (int p = tid; p < tile_n; p += kSortThreads) {
        const unsigned long long x = s_items[p];
        const uint32_t d = (item_key(x) >> shift) & (kRadix - 1);
        dst[(uint32_t)(s_gbase[d] + (uint32_t)p)] = x;
    }
}

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

// Number of segment heads (first item, or key differs from the previous) per range.
__global__ void __launch_bounds__(kSegThreads)
    seg_count(const unsigned long long *__restrict__ items, int64_t n, int W,
              uint32_t *__restrict__ wcount)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= W)
        return;
    int64_t a, b;
    range_of(n, w, W, a, b);
    uint32_t cnt = 0;
    for (int64_t c0 = a; c0 < b; c0 += 32) {
        const int64_t i = c0 + lane;
        const bool live = i < b;
        const uint32_t key = live ? item_key(__ldg(items + i)) : 0u;
        const uint32_t prev = (live && i > 0) ? item_key(__ldg(items + i - 1)) : ~key;
        cnt += __popc(__ballot_sync(kFull, live && key != prev));
    }
    if (lane == 0)
        wcount[w] = cnt;
}

// Exclusive scan of the per-range head counts (one block); total = U.
__global__ void __launch_bounds__(1024)
    seg_scan(const uint32_t *__restrict__ wcount, int W, uint32_t *__restrict__ wbase,
             int32_t *__restrict__ num_unique)
{
    __shared__ uint32_t s_warp[32];
    uint32_t carry = 0;
    for (int w0 = 0; w0 < W; w0 += 1024) {
        const int w = w0 + threadIdx.x;
        const uint32_t v = w < W ? wcount[w] : 0u;
        uint32_t tot;
        const uint32_t ex = block_exclusive_scan(v, s_warp, &tot);
        if (w < W)
            wbase[w] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0)
        *num_unique = (int32_t)carry;
}

// 8 consecutive values of row j, group col (8 * col .. 8 * col + 7), as fp32.
template <int DT>
__device__ __forceinline__ void load_group(const void *__restrict__ dout, uint32_t j, int dim,
                                           int col, uint4 &lo, uint4 &hi)
{
    if constexpr (DT == ENGRAM_F32) {
        const uint4 *p = (const uint4 *)((const float *)dout + (size_t)j * dim) + 2 * col;
        lo = ld_stream(p);
        hi = ld_stream(p + 1);
    } else {
        const uint4 *p = (const uint4 *)((const uint16_t *)dout + (size_t)j * dim) + col;
        lo = ld_stream(p);
    }
}

template <int DT>
__device__ __forceinline__ void add_group(double (&acc)[8], const uint4 &lo, const uint4 &hi)
{
    if constexpr (DT == ENGRAM_F32) {
        acc[0] += (double)__uint_as_float(lo.x);
        acc[1] += (double)__uint_as_float(lo.y);
        acc[2] += (double)__uint_as_float(lo.z);
        acc[3] += (double)__uint_as_float(lo.w);
        acc[4] += (double)__uint_as_float(hi.x);
        acc[5] += (double)__uint_as_float(hi.y);
        acc[6] += (double)__uint_as_float(hi.z);
        acc[7] += (double)__uint_as_float(hi.w);
    } else if constexpr (DT == ENGRAM_BF16) {
        const uint32_t w[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc[2 * q] += (double)__uint_as_float(w[q] << 16);
            acc[2 * q + 1] += (double)__uint_as_float(w[q] & 0xffff0000u);
        }
    } else {
        const uint32_t w[4] = {lo.x, lo.y, lo.z, lo.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            __half2 h2;
            memcpy(&h2, &w[q], 4);
            const float2 f = __half22float2(h2);
            acc[2 * q] += (double)f.x;
            acc[2 * q + 1] += (double)f.y;
        }
    }
}

// Row gradient: the fp64 sums rounded once to fp32.
template <int G>
__device__ __forceinline__ void store_groups(float *__restrict__ dst, const double (&acc)[G][8],
                                             int lane, int CV)
{
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int col = lane + 32 * g;
        if (col < CV) {
            float4 *p = (float4 *)(dst + 8 * col);
            st_stream(p, make_float4((float)acc[g][0], (float)acc[g][1], (float)acc[g][2],
                                     (float)acc[g][3]));
            st_stream(p + 1, make_float4((float)acc[g][4], (float)acc[g][5], (float)acc[g][6],
                                         (float)acc[g][7]));
        }
    }
}

// Partial sum of a segment piece, kept in fp64.
template <int G>
__device__ __forceinline__ void store_partial(double *__restrict__ dst, const double (&acc)[G][8],
                                              int lane, int CV)
{
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int col = lane + 32 * g;
        if (col < CV) {
            double2 *p = (double2 *)(dst + 8 * col);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                p[k] = make_double2(acc[g][2 * k], acc[g][2 * k + 1]);
        }
    }
}

// Segmented fp32 sums over one contiguous range of sorted items per warp.
// G = 8-value column groups per lane (dim <= 256 * G).
template <int DT, int G>
__global__ void __launch_bounds__(kSegThreads)
    seg_reduce(const unsigned long long *__restrict__ items, int64_t n, int W,
               const uint32_t *__restrict__ wbase, const void *__restrict__ dout, int dim,
               int32_t *__restrict__ uniq, float *__restrict__ grads, double *__restrict__ pb,
               double *__restrict__ pe, SegMeta *__restrict__ meta)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= W)
        return;
    int64_t a, b;
    range_of(n, w, W, a, b);
    const int CV = dim >> 3;

    double acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int q = 0; q < 8; ++q)
            acc[g][q] = 0.0;

    // If the range opens in the middle of a segment that began earlier, its
    // first head (if any) closes that piece, which goes to pb.
    int32_t u = (int32_t)wbase[w] - 1; // index of the open segment
    uint32_t cur_key = 0;
    bool open_here = false; // the open segment's head lies in this range
    int32_t pb_ends = 0;

    for (int64_t c0 = a; c0 < b; c0 += 32) {
        const int64_t i = c0 + lane;
        const bool live = i < b;
        const unsigned long long it = live ? __ldg(items + i) : 0ull;
        const uint32_t key = item_key(it);
        const uint32_t j = (uint32_t)it;
        uint32_t prev = __shfl_up_sync(kFull, key, 1);
        if (lane == 0)
            prev = c0 > 0 ? item_key(__ldg(items + c0 - 1)) : ~key;
        const uint32_t heads = __ballot_sync(kFull, live && key != prev);
        const int nlive = (int)min64(32, b - c0);

        for (int e0 = 0; e0 < nlive; e0 += kSegPrefetch) {
            uint4 lo[kSegPrefetch][G], hi[kSegPrefetch][G];
#pragma unroll
            for (int q = 0; q < kSegPrefetch; ++q) {
                const int e = e0 + q;
                const uint32_t jj = __shfl_sync(kFull, j, e);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const int col = lane + 32 * g;
                    lo[q][g] = hi[q][g] = make_uint4(0, 0, 0, 0);
                    if (e < nlive && col < CV)
                        load_group<DT>(dout, jj, dim, col, lo[q][g], hi[q][g]);
                }
            }
#pragma unroll
            for (int q = 0; q < kSegPrefetch; ++q) {
                const int e = e0 + q;
                if (e < nlive) {
                    if ((heads >> e) & 1u) {
                        if (c0 + e > a) {
                            // close the segment that ends just before this head
                            if (open_here) {
                                store_groups<G>(grads + (size_t)u * dim, acc, lane, CV);
                                if (lane == 0)
                                    uniq[u] = (int32_t)cur_key;
                            } else {
                                store_partial<G>(pb + (size_t)w * dim, acc, lane, CV);
                                pb_ends = 1;
                            }
                        }
                        ++u;
                        cur_key = __shfl_sync(kFull, key, e);
                        open_here = true;
#pragma unroll
                        for (int g = 0; g < G; ++g)
#pragma unroll
                            for (int k = 0; k < 8; ++k)
                                acc[g][k] = 0.0;
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        add_group<DT>(acc[g], lo[q][g], hi[q][g]);
                }
            }
        }
    }

    // The range's last segment: does it go on past b?
    const bool cont = b < n && item_key(__ldg(items + b)) == item_key(__ldg(items + b - 1));
    int32_t pe_valid = 0;
    if (open_here) {
        if (cont) {
            store_partial<G>(pe + (size_t)w * dim, acc, lane, CV);
            pe_valid = 1;
        } else {
            store_groups<G>(grads + (size_t)u * dim, acc, lane, CV);
            if (lane == 0)
                uniq[u] = (int32_t)cur_key;
        }
    } else {
        // no head in the range: it is one piece of a segment begun earlier
        store_partial<G>(pb + (size_t)w * dim, acc, lane, CV);
        pb_ends = cont ? 0 : 1;
    }
    if (lane == 0)
        meta[w] = SegMeta{pe_valid, u, (int32_t)cur_key, pb_ends};
}

// One warp per segment that crosses range boundaries: its head piece plus the
// following ranges' pieces, in range order.
template <int G>
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
    const int CV = dim >> 3;
    double acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int col = lane + 32 * g;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            acc[g][k] = col < CV ? pe[(size_t)w * dim + 8 * col + k] : 0.0;
    }
    for (int64_t w2 = w + 1; w2 < W; ++w2) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const int col = lane + 32 * g;
            if (col < CV) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    acc[g][k] += pb[(size_t)w2 * dim + 8 * col + k];
            }
        }
        if (meta[w2].pb_ends)
            break;
    }
    store_groups<G>(grads + (size_t)m.pe_u * dim, acc, lane, CV);
    if (lane == 0)
        uniq[m.pe_u] = m.pe_key;
}

} // namespace bwd
} // namespace engram
