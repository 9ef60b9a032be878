// radix_sort.cuh -- stable LSD radix sort of the backward's (row, lookup) pairs.
//
// The pairs (idx[j], j) are packed as 64-bit items key << 32 | j and sorted by
// key, 8 bits per pass, ceil(bits(table_rows - 1) / 8) passes. Because the
// items start in j order and every pass is stable, equal keys end up in
// ascending j.
//
// Each pass has two phases over tiles of 256 * ITEMS items (ITEMS <= 8 pairs
// per thread, chosen per sort by the host so that the busiest SM holds as few
// pairs as possible):
//   count    a tile's digit counts are stored (tile-major, tile_cnt[tile][d])
//            and added into per-group sums (group_cnt[group][d], 32 tiles per
//            group; the adds commute, so the sums are deterministic);
//   scatter  a tile ranks its items stably in shared memory (per-warp digit
//            counters, peers found with one ballot per digit bit), takes each
//            digit's global offset as
//              sum of all earlier digits' totals
//              + that digit's group sums before the tile's group
//              + that digit's tile counts earlier in the group
//            (a few dozen independent, coalesced loads per thread), and writes
//            the tile out in contiguous runs staged through shared memory.
// No tile ever waits on another tile's result, so there is no serial prefix
// chain across tiles.
//
// radix_sort_coop runs every phase of every pass in one cooperative launch:
// each resident block takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... and
// the phases are separated by a grid barrier on one arrival counter (bounded
// wait; a timeout raises ENGRAM_DEVERR_SORT_TIMEOUT instead of hanging). Data written by other blocks
// in the same launch is read through L2 (ld.global.cg), never through the
// non-coherent load path. radix_count / radix_scatter run the same phases as
// separate launches where cooperative launch is unavailable.
#pragma once

#include "common.cuh"

namespace engram {
namespace bwd {

constexpr int kSortThreads = 256;
constexpr int kSortItemsMax = 8; // pairs per thread of the largest tile (2048 pairs)
constexpr int kRadixBits = 8;
constexpr int kRadix = 1 << kRadixBits;
constexpr int kMaxPasses = 4; // keys below 2^32
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kTilesPerGroup = 32;
constexpr uint32_t kBarrierSpin = 1u << 22; // polls (~64 ns apart) before a barrier gives up
static_assert(kRadix == kSortThreads, "one thread per digit");

__device__ __forceinline__ uint32_t item_key(uint64_t it) { return (uint32_t)(it >> 32); }

template <int ITEMS> struct SortSmem {
    static constexpr int kTile = kSortThreads * ITEMS;
    uint32_t whist[kSortWarps][kRadix];
    uint32_t tstart[kRadix];
    uint32_t gbase[kRadix];
    uint32_t cnt[kRadix];
    uint32_t warp[32];
    unsigned long long warp2[32];
    unsigned long long items[kTile];
    int flag;
};

// Item i of a pass: pass 0 forms it from the int32 index, later passes read it.
// COHERENT loads go through L2 only (needed when another block of the same
// launch wrote the data); otherwise the read-only path is used.
template <bool COHERENT>
__device__ __forceinline__ uint64_t load_item(const void *__restrict__ src, bool first, int64_t i)
{
    if (first) {
        const int32_t *p = (const int32_t *)src + i;
        const uint32_t key = (uint32_t)(COHERENT ? __ldcg(p) : __ldg(p));
        return ((uint64_t)key << 32) | (uint32_t)i;
    }
    const unsigned long long *p = (const unsigned long long *)src + i;
    return COHERENT ? __ldcg(p) : __ldg(p);
}

template <bool COHERENT>
__device__ __forceinline__ uint32_t load_u32(const uint32_t *p)
{
    return COHERENT ? __ldcg(p) : __ldg(p);
}

// Lanes of the warp whose digit equals this lane's (valid lanes only).
__device__ __forceinline__ uint32_t digit_peers(uint32_t dg, bool valid)
{
    uint32_t peers = __ballot_sync(kFull, valid);
#pragma unroll
    for (int bit = 0; bit < kRadixBits; ++bit) {
        const bool on = (dg >> bit) & 1u;
        const uint32_t bal = __ballot_sync(kFull, on);
        peers &= on ? bal : ~bal;
    }
    return peers;
}

// Count phase of one tile. Pass 0 also flags keys outside [0, rows).
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void count_tile(SortSmem<ITEMS> &sm, const void *src, bool first, int64_t n,
                                           int shift, uint32_t rows, int tile,
                                           uint32_t *tile_cnt, uint32_t *group_cnt)
{
    const int tid = threadIdx.x, lane = tid & 31;
    sm.cnt[tid] = 0;
    __syncthreads();
    const int64_t base = (int64_t)tile * SortSmem<ITEMS>::kTile;
    uint32_t key[ITEMS];
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const int64_t i = base + r * kSortThreads + tid;
        key[r] = i < n ? item_key(load_item<COHERENT>(src, first, i)) : 0u;
    }
    bool bad = false;
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const bool valid = base + r * kSortThreads + tid < n;
        if (first && valid && key[r] >= rows)
            bad = true;
        // one shared-memory add per distinct digit in the warp, so runs of a
        // hot key do not serialise on one counter
        const uint32_t dg = (key[r] >> shift) & (kRadix - 1);
        const uint32_t peers = digit_peers(dg, valid);
        if (valid && lane == __ffs(peers) - 1)
            atomicAdd(&sm.cnt[dg], (uint32_t)__popc(peers));
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    __syncthreads();
    const uint32_t c = sm.cnt[tid];
    tile_cnt[(size_t)tile * kRadix + tid] = c;
    if (c)
        atomicAdd(&group_cnt[(size_t)(tile / kTilesPerGroup) * kRadix + tid], c);
    __syncthreads(); // sm.cnt free for the next tile
}

// Loads the tile's items and ranks them stably: rank[r] is item r's position
// among the items of its digit in its warp, and sm.whist[w][d] ends up as the
// number of items of digit d in warp w. Pass 0 also flags keys outside the table.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void rank_tile(SortSmem<ITEMS> &sm, const void *src, bool first,
                                          int64_t n, int shift, uint32_t rows, int tile,
                                          uint64_t (&it)[ITEMS], uint32_t (&rank)[ITEMS])
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int k = tid; k < kSortWarps * kRadix; k += kSortThreads)
        (&sm.whist[0][0])[k] = 0;
    const int64_t wbase = (int64_t)tile * SortSmem<ITEMS>::kTile + (int64_t)wid * (32 * ITEMS);
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        it[r] = i < n ? load_item<COHERENT>(src, first, i) : 0ull;
    }
    __syncthreads(); // whist zeroed
    bool bad = false;
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const bool valid = wbase + r * 32 + lane < n;
        if (first && valid && item_key(it[r]) >= rows)
            bad = true;
        const uint32_t dg = (item_key(it[r]) >> shift) & (kRadix - 1);
        const uint32_t peers = digit_peers(dg, valid);
        const int leader = valid ? __ffs(peers) - 1 : lane;
        uint32_t cnt = 0;
        if (valid && lane == leader) {
            cnt = sm.whist[wid][dg];
            sm.whist[wid][dg] = cnt + __popc(peers);
        }
        cnt = __shfl_sync(kFull, cnt, leader);
        rank[r] = cnt + __popc(peers & lt);
        __syncwarp();
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    __syncthreads();
}

// Thread d: turns sm.whist[.][d] into per-warp exclusive offsets and returns
// the tile's count of digit d.
template <int ITEMS> __device__ __forceinline__ uint32_t tile_digit_count(SortSmem<ITEMS> &sm)
{
    const int d = threadIdx.x;
    uint32_t tcount = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
        const uint32_t c = sm.whist[w][d];
        sm.whist[w][d] = tcount;
        tcount += c;
    }
    return tcount;
}

// Stores a tile's digit counts (tile-major) and adds them into its group's sums.
__device__ __forceinline__ void publish_counts(int tile, uint32_t tcount, uint32_t *tile_cnt,
                                               uint32_t *group_cnt)
{
    const int d = threadIdx.x;
    tile_cnt[(size_t)tile * kRadix + d] = tcount;
    if (tcount)
        atomicAdd(&group_cnt[(size_t)(tile / kTilesPerGroup) * kRadix + d], tcount);
}

// Once every tile of the pass has published its counts: sm.tstart[d] = the
// start of digit d = threadIdx.x in the tile, sm.gbase[d] = its global start
// minus that. tcount is digit d's count in the tile.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void tile_offsets(SortSmem<ITEMS> &sm, int tile, uint32_t tcount,
                                             const uint32_t *tile_cnt,
                                             const uint32_t *group_cnt, int ngroups)
{
    // Counts are tile- and group-major, so each load instruction reads 32
    // consecutive digits; the loops are unrolled so the loads are in flight
    // together.
    const int d = threadIdx.x;
    const int grp = tile / kTilesPerGroup;
    uint32_t excl = 0, total = 0;
    for (int g0 = 0; g0 < ngroups; g0 += 8) {
        uint32_t c[8];
#pragma unroll
        for (int q = 0; q < 8; ++q)
            c[q] = g0 + q < ngroups
                       ? load_u32<COHERENT>(group_cnt + (size_t)(g0 + q) * kRadix + d)
                       : 0u;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            total += c[q];
            if (g0 + q < grp)
                excl += c[q];
        }
    }
    {
        const int t0 = grp * kTilesPerGroup;
        uint32_t c[kTilesPerGroup];
#pragma unroll
        for (int q = 0; q < kTilesPerGroup; ++q)
            c[q] = t0 + q < tile ? load_u32<COHERENT>(tile_cnt + (size_t)(t0 + q) * kRadix + d)
                                 : 0u;
#pragma unroll
        for (int q = 0; q < kTilesPerGroup; ++q)
            excl += c[q];
    }

    // One scan over digits gives both the tile-local start (low half) and the
    // start of the digit among all digits (high half).
    const unsigned long long both = block_exclusive_scan64(
        ((unsigned long long)total << 32) | tcount, (unsigned long long *)sm.warp2);
    const uint32_t tstart = (uint32_t)both, dbase = (uint32_t)(both >> 32);
    sm.tstart[d] = tstart;
    sm.gbase[d] = dbase + excl - tstart;
    __syncthreads();
}

// Writes a ranked tile to its sorted positions, once every tile of the pass
// has published its counts. tcount is digit threadIdx.x's count in the tile.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void place_tile(SortSmem<ITEMS> &sm, unsigned long long *dst,
                                           int64_t n, int shift, int tile, uint32_t tcount,
                                           const uint64_t (&it)[ITEMS],
                                           const uint32_t (&rank)[ITEMS],
                                           const uint32_t *tile_cnt, const uint32_t *group_cnt,
                                           int ngroups)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    tile_offsets<COHERENT>(sm, tile, tcount, tile_cnt, group_cnt, ngroups);

    const int64_t wbase = (int64_t)tile * SortSmem<ITEMS>::kTile + (int64_t)wid * (32 * ITEMS);
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        if (wbase + r * 32 + lane < n) {
            const uint32_t dg = (item_key(it[r]) >> shift) & (kRadix - 1);
            sm.items[sm.tstart[dg] + sm.whist[wid][dg] + rank[r]] = it[r];
        }
    }
    __syncthreads();
    const int64_t base = (int64_t)tile * SortSmem<ITEMS>::kTile;
    const int tile_n = (int)min64(SortSmem<ITEMS>::kTile, n - base);
    for (int p = tid; p < tile_n; p += kSortThreads) {
        const unsigned long long x = sm.items[p];
        const uint32_t dg = (item_key(x) >> shift) & (kRadix - 1);
        dst[(uint32_t)(sm.gbase[dg] + (uint32_t)p)] = x;
    }
    __syncthreads(); // shared memory free for the next tile
}

// Scatter phase of one tile after a separate count phase: rank, then place.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void scatter_tile(SortSmem<ITEMS> &sm, const void *src, bool first,
                                             unsigned long long *dst, int64_t n, int shift,
                                             int tile, const uint32_t *tile_cnt,
                                             const uint32_t *group_cnt, int ngroups)
{
    uint64_t it[ITEMS];
    uint32_t rank[ITEMS];
    // (the count phase has already checked the keys against the table)
    rank_tile<COHERENT>(sm, src, first, n, shift, 0xffffffffu, tile, it, rank);
    const uint32_t tcount = tile_digit_count(sm);
    place_tile<COHERENT>(sm, dst, n, shift, tile, tcount, it, rank, tile_cnt, group_cnt,
                         ngroups);
}

// Count phase of the one-launch sort when tiles outnumber the resident
// blocks (a block cannot keep its tiles' items and ranks across the barrier):
// ranks the tile, publishes its digit counts and writes it back ordered by
// digit, stably, into its own region of `ordered`, so that the place phase
// need not rank it again. `ordered` may be `src` itself (the tile region is
// read before it is written, by this block alone).
template <int ITEMS>
__device__ __forceinline__ void count_order_tile(SortSmem<ITEMS> &sm, const void *src, bool first,
                                                 int64_t n, int shift, uint32_t rows, int tile,
                                                 uint32_t *tile_cnt, uint32_t *group_cnt,
                                                 unsigned long long *ordered)
{
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    uint64_t it[ITEMS];
    uint32_t rank[ITEMS];
    rank_tile<true>(sm, src, first, n, shift, rows, tile, it, rank);
    const uint32_t tcount = tile_digit_count(sm);
    publish_counts(tile, tcount, tile_cnt, group_cnt);
    sm.tstart[tid] = block_exclusive_scan(tcount, sm.warp, nullptr);
    __syncthreads();
    const int64_t base = (int64_t)tile * SortSmem<ITEMS>::kTile;
    const int64_t wbase = base + (int64_t)wid * (32 * ITEMS);
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        if (wbase + r * 32 + lane < n) {
            const uint32_t dg = (item_key(it[r]) >> shift) & (kRadix - 1);
            sm.items[sm.tstart[dg] + sm.whist[wid][dg] + rank[r]] = it[r];
        }
    }
    __syncthreads();
    const int tile_n = (int)min64(SortSmem<ITEMS>::kTile, n - base);
    for (int q = tid; q < tile_n; q += kSortThreads)
        ordered[base + q] = sm.items[q];
    __syncthreads(); // shared memory free for the next tile
}

// Place phase for a tile that count_order_tile left ordered by digit: each
// run of one digit goes to that digit's global offsets.
template <int ITEMS>
__device__ __forceinline__ void place_ordered_tile(SortSmem<ITEMS> &sm,
                                                   const unsigned long long *ordered,
                                                   unsigned long long *dst, int64_t n, int shift,
                                                   int tile, const uint32_t *tile_cnt,
                                                   const uint32_t *group_cnt, int ngroups)
{
    const int tid = threadIdx.x;
    const uint32_t tcount = __ldcg(tile_cnt + (size_t)tile * kRadix + tid);
    tile_offsets<true>(sm, tile, tcount, tile_cnt, group_cnt, ngroups);
    const int64_t base = (int64_t)tile * SortSmem<ITEMS>::kTile;
    const int tile_n = (int)min64(SortSmem<ITEMS>::kTile, n - base);
    for (int q = tid; q < tile_n; q += kSortThreads) {
        const unsigned long long x = __ldcg(ordered + base + q);
        const uint32_t dg = (item_key(x) >> shift) & (kRadix - 1);
        dst[(uint32_t)(sm.gbase[dg] + (uint32_t)q)] = x;
    }
    __syncthreads(); // shared memory free for the next tile
}

// ----------------------------------------------- one launch per phase

template <bool FIRST, int ITEMS>
__global__ void __launch_bounds__(kSortThreads)
    radix_count(const void *__restrict__ src, int64_t n, int shift, uint32_t rows,
                uint32_t *__restrict__ tile_cnt, uint32_t *__restrict__ group_cnt)
{
    __shared__ SortSmem<ITEMS> sm;
    count_tile<false>(sm, src, FIRST, n, shift, rows, blockIdx.x, tile_cnt, group_cnt);
}

template <bool FIRST, int ITEMS>
__global__ void __launch_bounds__(kSortThreads)
    radix_scatter(const void *__restrict__ src, unsigned long long *__restrict__ dst,
                  int64_t n, int shift, const uint32_t *__restrict__ tile_cnt,
                  const uint32_t *__restrict__ group_cnt, int ngroups)
{
    __shared__ SortSmem<ITEMS> sm;
    scatter_tile<false>(sm, src, FIRST, dst, n, shift, blockIdx.x, tile_cnt, group_cnt,
                        ngroups);
}

// ------------------------------------------------ one cooperative launch

struct SortArgs {
    const int32_t *idx;
    unsigned long long *a, *b; // ping-pong item buffers; pass p writes (p even ? a : b)
    int64_t n;
    uint32_t rows;
    int passes, ntiles, ngroups;
    uint32_t *tile_cnt;  // [ntiles][256], rewritten every pass
    uint32_t *group_cnt; // [passes][ngroups][256], zero on entry
    unsigned *barrier;   // grid-barrier arrival counter; zero on entry
    uint32_t spin_limit; // polls before a grid-barrier wait gives up (<= kBarrierSpin)
};

// Grid-wide barrier among co-resident blocks on one arrival counter that only
// grows: barrier k of the launch is passed once the counter reaches
// k * gridDim.x. Thread 0 of each block arrives with one acquire-release add
// and, unless it was the last to arrive, polls the counter with acquire loads
// (bounded; giving up raises ENGRAM_DEVERR_SORT_TIMEOUT and returns false).
// The block's other threads wait at __syncthreads, which orders their later
// reads after thread 0's acquire. The counter is zero at launch.
__device__ __forceinline__ bool grid_barrier(unsigned *bar, unsigned &gen, int &flag,
                                             uint32_t spin_limit)
{
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned target = (gen + 1) * gridDim.x;
        unsigned before;
        asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                     : "=r"(before)
                     : "l"(bar)
                     : "memory");
        bool ok = true;
        if (before + 1 < target) {
            uint32_t spins = 0;
            while (ld_acquire_u32(bar) < target) {
                if (++spins > spin_limit) {
                    raise_device_error(ENGRAM_DEVERR_SORT_TIMEOUT);
                    ok = false;
                    break;
                }
                __nanosleep(64);
            }
        }
        flag = ok;
    }
    __syncthreads();
    gen += 1;
    return flag != 0;
}

// Four blocks per SM keep 592 tiles (1.2M pairs at ITEMS = 8) resident on a
// 148-SM B200.
template <int ITEMS> __global__ void __launch_bounds__(kSortThreads, 4) radix_sort_coop(SortArgs a)
{
    __shared__ SortSmem<ITEMS> sm;
    unsigned gen = 0;
    if (a.ntiles <= (int)gridDim.x) {
        // One tile per block: rank once, keep the items and their ranks in
        // registers (and the per-warp offsets in shared memory) across the
        // barrier, then place them.
        const int tile = blockIdx.x;
        const bool has = tile < a.ntiles;
        for (int pass = 0; pass < a.passes; ++pass) {
            const bool first = pass == 0;
            const void *src = first ? (const void *)a.idx : (pass % 2 == 1 ? a.a : a.b);
            unsigned long long *dst = pass % 2 == 0 ? a.a : a.b;
            uint32_t *gc = a.group_cnt + (size_t)pass * a.ngroups * kRadix;
            const int shift = pass * kRadixBits;
            uint64_t it[ITEMS];
            uint32_t rank[ITEMS];
            uint32_t tcount = 0;
            if (has) {
                rank_tile<true>(sm, src, first, a.n, shift, a.rows, tile, it, rank);
                tcount = tile_digit_count(sm);
                publish_counts(tile, tcount, a.tile_cnt, gc);
            }
            if (!grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
                return;
            if (has)
                place_tile<true>(sm, dst, a.n, shift, tile, tcount, it, rank, a.tile_cnt, gc,
                                 a.ngroups);
            if (pass + 1 < a.passes && !grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
                return;
        }
        return;
    }
    // More tiles than resident blocks: each tile is ranked once, in the count
    // phase, and left ordered by digit in `ordered` (the pass's own input from
    // the second pass on; the other item buffer on the first, whose input is
    // idx), from where the place phase moves it.
    for (int pass = 0; pass < a.passes; ++pass) {
        const bool first = pass == 0;
        const void *src = first ? (const void *)a.idx : (pass % 2 == 1 ? a.a : a.b);
        unsigned long long *dst = pass % 2 == 0 ? a.a : a.b;
        unsigned long long *ordered = first ? a.b : (pass % 2 == 1 ? a.a : a.b);
        uint32_t *gc = a.group_cnt + (size_t)pass * a.ngroups * kRadix;
        const int shift = pass * kRadixBits;
        for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x)
            count_order_tile(sm, src, first, a.n, shift, a.rows, tile, a.tile_cnt, gc, ordered);
        if (!grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
            return;
        for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x)
            place_ordered_tile(sm, ordered, dst, a.n, shift, tile, a.tile_cnt, gc, a.ngroups);
        if (pass + 1 < a.passes && !grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
            return;
    }
}

} // namespace bwd
} // namespace engram
