// radix_sort.cuh -- stable LSD radix sort of the backward's (row, lookup) pairs.
//
// The pairs (idx[j], j) are packed as 64-bit items key << 32 | j and sorted by
// key. Because the items enter each pass in ascending j and every pass is
// stable, equal keys end up in ascending j.
//
// Segments. A sort covers S segments of L positions each (n = S * L) and
// sorts every segment on its own; the segments are laid out one after the
// other. The plain sort is one segment holding all n lookups. The sort by
// head uses the structure of the hash's output (engram API page,
// Qwen3_8_FlashNextNGramEmbedding._hash_input_ids): lookup j = t * H + h of
// token t and head h always lies in head h's own slice [o_h, o_h + p_h) of the
// table, the slices are disjoint and ascend with h, and every head holds
// exactly T lookups. So segment h takes head h's lookups (position h * T + t
// holds lookup t * H + h), its keys are sorted as key - o_h, which needs only
// bits(p_h - 1) bits (25 on the page's table, against 29 for the whole key),
// and the concatenated segments are the whole sort. The last pass adds o_h
// back, so both forms leave the same items.
//
// Passes take digits of up to 9 bits (the key's bits spread evenly over the
// fewest passes), least significant first. Each pass has two phases over
// tiles of 256 * ITEMS items (ITEMS = 4..8, chosen per sort by the host);
// a tile never spans two segments:
//   count    a tile's digit counts are stored (tile_cnt[tile][d]) and added
//            into per-group sums (group_cnt[pass][group][d], groups of 32
//            tiles inside one segment; the adds commute, so the sums are
//            deterministic);
//   place    a tile ranks its items stably in shared memory (per-warp digit
//            counters, peers found with one ballot per digit bit), takes each
//            digit's position in its segment as
//              sum of the earlier digits' totals in the segment
//              + that digit's group sums before the tile's group
//              + that digit's tile counts earlier in the group
//            (independent, coalesced loads), and writes the tile out in
//            contiguous runs staged through shared memory.
// No tile ever waits on another tile's result, so there is no serial prefix
// chain across tiles. The last pass always writes buffer `a`, so the reduce
// finds the sorted items in one place whatever the number of passes.
//
// radix_sort_coop runs every phase of every pass in one cooperative launch:
// each resident block takes tiles blockIdx.x, blockIdx.x + gridDim.x, ... and
// the phases are separated by a grid barrier on one arrival counter (bounded
// wait; a timeout raises ENGRAM_DEVERR_SORT_TIMEOUT instead of hanging). Data
// written by other blocks in the same launch is read through L2
// (ld.global.cg), never through the non-coherent load path. radix_count /
// radix_scatter run the same phases as separate launches where cooperative
// launch is unavailable.
#pragma once

#include "common.cuh"

namespace engram {
namespace bwd {

constexpr int kSortThreads = 256;
constexpr int kSortItemsMin = 4;
constexpr int kSortItemsMax = 8;   // pairs per thread of the largest tile (2048 pairs)
constexpr int kDigitBitsMax = 9;
constexpr int kRadixMax = 1 << kDigitBitsMax;
constexpr int kMaxPasses = 4;      // keys below 2^32 at <= 9 bits per pass
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kTilesPerGroup = 32;
constexpr int kMaxSegments = ENGRAM_MAX_HEADS;
constexpr uint32_t kBarrierSpin = 1u << 22; // polls (~64 ns apart) before a barrier gives up
static_assert(kRadixMax == 2 * kSortThreads, "at most two digits per thread");

struct SortArgs {
    const int32_t *idx;
    unsigned long long *a, *b; // ping-pong item buffers; the last pass writes a
    int64_t n;                 // S * L
    int64_t L;                 // positions per segment
    int S;                     // segments
    int passes;
    int bits[kMaxPasses];      // digit width of each pass, least significant first
    int tps, gps;              // tiles and 32-tile groups per segment
    int ntiles, ngroups;       // S * tps, S * gps
    uint32_t *tile_cnt;        // [ntiles][kRadixMax], rewritten every pass
    uint32_t *group_cnt;       // [passes][ngroups][kRadixMax], zero on entry
    unsigned *barrier;         // grid-barrier arrival counter; zero on entry
    uint32_t spin_limit;       // polls before a grid-barrier wait gives up
    int32_t off[kMaxSegments]; // segment s holds keys off[s] .. off[s] + size[s] - 1
    uint32_t size[kMaxSegments];
    bool pad;                  // a negative index is an absent lookup: key size[s], not an error
};

__device__ __forceinline__ uint32_t item_key(uint64_t it) { return (uint32_t)(it >> 32); }

// One pass: its digit is bits [shift, shift + bits) of the (segment-relative) key.
struct PassInfo {
    int shift, bits, ndig, dpt; // dpt: digits per thread (1, or 2 above 8 bits)
    bool first, last;
};

__device__ __forceinline__ PassInfo pass_info(const SortArgs &a, int p)
{
    PassInfo q;
    q.shift = 0;
    for (int k = 0; k < p; ++k)
        q.shift += a.bits[k];
    q.bits = a.bits[p];
    q.ndig = 1 << q.bits;
    q.dpt = q.ndig > kSortThreads ? 2 : 1;
    q.first = p == 0;
    q.last = p == a.passes - 1;
    return q;
}

__device__ __forceinline__ uint32_t digit_of(uint64_t x, const PassInfo &P)
{
    return (item_key(x) >> P.shift) & (uint32_t)(P.ndig - 1);
}

// Pass p writes `out_buffer(a, p)` and reads the previous pass's output; the
// parity is set so that the last pass writes a.
__device__ __forceinline__ unsigned long long *out_buffer(const SortArgs &a, int p)
{
    return ((a.passes - 1 - p) & 1) == 0 ? a.a : a.b;
}

struct TileGeom {
    int seg;       // segment of the tile
    int k;         // tile index inside the segment
    int64_t begin; // first position
    int count;     // positions (the segment's last tile may be short)
};

__device__ __forceinline__ TileGeom tile_geom(const SortArgs &a, int tile, int tile_items)
{
    TileGeom g;
    g.seg = tile / a.tps;
    g.k = tile - g.seg * a.tps;
    const int64_t lo = (int64_t)g.k * tile_items;
    g.begin = (int64_t)g.seg * a.L + lo;
    g.count = (int)min64(tile_items, a.L - lo);
    return g;
}

template <int ITEMS> struct SortSmem {
    static constexpr int kTile = kSortThreads * ITEMS;
    uint32_t whist[kSortWarps][kRadixMax];
    uint32_t tstart[kRadixMax];
    uint32_t gbase[kRadixMax];
    uint32_t cnt[kRadixMax];
    uint32_t warp[32];
    unsigned long long warp2[32];
    unsigned long long items[kTile];
    int flag;
};

// Item at position i (0 <= i < count) of a tile. The first pass forms it from
// the int32 index of lookup j = (k * TILE + i) * S + seg, keyed relative to
// the segment's first row; later passes read the previous pass's output.
// COHERENT loads go through L2 only (needed when another block of the same
// launch wrote the data).
// The first pass's item of lookup j: its key relative to the segment, or the
// segment's size for an absent lookup (negative index, when a.pad); `bad`
// is set for an index outside the segment's rows.
__device__ __forceinline__ uint64_t first_item(const SortArgs &a, int seg, int64_t j, bool &bad)
{
    const int32_t v = __ldg(a.idx + j);
    uint32_t key;
    if (a.pad && v < 0) {
        key = a.size[seg];
    } else {
        key = (uint32_t)v - (uint32_t)a.off[seg];
        bad |= key >= a.size[seg];
    }
    return ((uint64_t)key << 32) | (uint32_t)j;
}

template <bool COHERENT>
__device__ __forceinline__ uint64_t load_item(const SortArgs &a, const void *__restrict__ src,
                                              bool first, const TileGeom &g, int tile_items,
                                              int i, bool &bad)
{
    if (first)
        return first_item(a, g.seg, ((int64_t)g.k * tile_items + i) * a.S + g.seg, bad);
    const unsigned long long *p = (const unsigned long long *)src + g.begin + i;
    return COHERENT ? __ldcg(p) : __ldg(p);
}

template <bool COHERENT>
__device__ __forceinline__ uint32_t load_u32(const uint32_t *p)
{
    return COHERENT ? __ldcg(p) : __ldg(p);
}

// Lanes of the warp whose digit equals this lane's (valid lanes only); `bits`
// is the same on every lane.
__device__ __forceinline__ uint32_t digit_peers(uint32_t dg, bool valid, int bits)
{
    uint32_t peers = __ballot_sync(kFull, valid);
#pragma unroll
    for (int bit = 0; bit < kDigitBitsMax; ++bit) {
        if (bit < bits) {
            const bool on = (dg >> bit) & 1u;
            const uint32_t bal = __ballot_sync(kFull, on);
            peers &= on ? bal : ~bal;
        }
    }
    return peers;
}

// Digit d of this thread's slot e (digits tid * dpt + e, consecutive per thread).
__device__ __forceinline__ int my_digit(const PassInfo &P, int e)
{
    return threadIdx.x * P.dpt + e;
}

// Count phase of one tile (separate-launch form). The first pass also flags
// keys outside their segment's rows.
template <int ITEMS>
__device__ __forceinline__ void count_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                           const void *src, const PassInfo &P, int tile,
                                           uint32_t *gc)
{
    constexpr int TILE = SortSmem<ITEMS>::kTile;
    const int tid = threadIdx.x, lane = tid & 31;
    const TileGeom g = tile_geom(a, tile, TILE);
    for (int d = tid; d < P.ndig; d += kSortThreads)
        sm.cnt[d] = 0;
    __syncthreads();
    uint32_t key[ITEMS];
    bool bad = false;
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const int i = r * kSortThreads + tid;
        key[r] = i < g.count ? item_key(load_item<false>(a, src, P.first, g, TILE, i, bad)) : 0u;
    }
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const bool valid = r * kSortThreads + tid < g.count;
        // one shared-memory add per distinct digit in the warp, so runs of a
        // hot key do not serialise on one counter
        const uint32_t dg = (key[r] >> P.shift) & (uint32_t)(P.ndig - 1);
        const uint32_t peers = digit_peers(dg, valid, P.bits);
        if (valid && lane == __ffs(peers) - 1)
            atomicAdd(&sm.cnt[dg], (uint32_t)__popc(peers));
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    __syncthreads();
    const int grp = g.seg * a.gps + g.k / kTilesPerGroup;
    for (int d = tid; d < P.ndig; d += kSortThreads) {
        const uint32_t c = sm.cnt[d];
        a.tile_cnt[(size_t)tile * kRadixMax + d] = c;
        if (c)
            atomicAdd(&gc[(size_t)grp * kRadixMax + d], c);
    }
    __syncthreads(); // sm.cnt free for the next tile
}

// Loads the tile's items and ranks them stably: rank[r] is item r's position
// among the items of its digit in its warp, and sm.whist[w][d] ends up as the
// number of items of digit d in warp w. The first pass also flags keys outside
// their segment's rows (check_keys).
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void rank_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                          const void *src, const PassInfo &P, const TileGeom &g,
                                          bool check_keys, uint64_t (&it)[ITEMS],
                                          uint32_t (&rank)[ITEMS])
{
    constexpr int TILE = SortSmem<ITEMS>::kTile;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int k = tid; k < (kSortWarps << P.bits); k += kSortThreads)
        sm.whist[k >> P.bits][k & (P.ndig - 1)] = 0;
    const int wbase = wid * (32 * ITEMS);
    const uint32_t lt = lanemask_lt();
    bool bad = false;
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const int i = wbase + r * 32 + lane;
        it[r] = i < g.count ? load_item<COHERENT>(a, src, P.first, g, TILE, i, bad) : 0ull;
    }
    bad = bad && check_keys;
    __syncthreads(); // whist zeroed
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        const bool valid = wbase + r * 32 + lane < g.count;
        const uint32_t dg = digit_of(it[r], P);
        const uint32_t peers = digit_peers(dg, valid, P.bits);
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

// For this thread's digits: turns sm.whist[.][d] into per-warp exclusive
// offsets and returns the tile's count of each digit in tcount[e].
template <int ITEMS>
__device__ __forceinline__ void tile_digit_count(SortSmem<ITEMS> &sm, const PassInfo &P,
                                                 uint32_t (&tcount)[2])
{
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        uint32_t run = 0;
        if (e < P.dpt && d < P.ndig) {
#pragma unroll
            for (int w = 0; w < kSortWarps; ++w) {
                const uint32_t c = sm.whist[w][d];
                sm.whist[w][d] = run;
                run += c;
            }
        }
        tcount[e] = run;
    }
}

// Stores a tile's digit counts and adds them into its group's sums.
__device__ __forceinline__ void publish_counts(const SortArgs &a, const PassInfo &P, int tile,
                                               const TileGeom &g, const uint32_t (&tcount)[2],
                                               uint32_t *gc)
{
    const int grp = g.seg * a.gps + g.k / kTilesPerGroup;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        if (e < P.dpt && d < P.ndig) {
            a.tile_cnt[(size_t)tile * kRadixMax + d] = tcount[e];
            if (tcount[e])
                atomicAdd(&gc[(size_t)grp * kRadixMax + d], tcount[e]);
        }
    }
}

// Tile-local start of each of this thread's digits into sm.tstart (an
// exclusive scan of the tile's digit counts over the block).
template <int ITEMS>
__device__ __forceinline__ void local_starts(SortSmem<ITEMS> &sm, const PassInfo &P,
                                             const uint32_t (&tcount)[2])
{
    uint32_t tstart = block_exclusive_scan(tcount[0] + tcount[1], sm.warp, nullptr);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        if (e < P.dpt && d < P.ndig) {
            sm.tstart[d] = tstart;
            tstart += tcount[e];
        }
    }
    __syncthreads();
}

// Ranks a tile, counts its digits (publishing the counts when `gc` is not
// null) and leaves its items in sm.items ordered by digit, stably; tcount[e]
// is the tile's count of this thread's digit e. Only the counts stay in
// registers afterwards.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void stage_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                           const void *src, const PassInfo &P, int tile,
                                           const TileGeom &g, bool check_keys, uint32_t *gc,
                                           uint32_t (&tcount)[2])
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint64_t it[ITEMS];
    uint32_t rank[ITEMS];
    rank_tile<COHERENT>(sm, a, src, P, g, check_keys, it, rank);
    tile_digit_count(sm, P, tcount);
    if (gc != nullptr)
        publish_counts(a, P, tile, g, tcount, gc);
    local_starts(sm, P, tcount);
    const int wbase = wid * (32 * ITEMS);
#pragma unroll
    for (int r = 0; r < ITEMS; ++r) {
        if (wbase + r * 32 + lane < g.count) {
            const uint32_t dg = digit_of(it[r], P);
            sm.items[sm.tstart[dg] + sm.whist[wid][dg] + rank[r]] = it[r];
        }
    }
    __syncthreads();
}

// Once every tile of the pass has published its counts: sm.gbase[d] = the
// position in the output of digit d's first item in the tile, minus
// sm.tstart[d] (which WITH_TSTART computes here from tcount; otherwise
// local_starts already has). tcount[e] is the tile's count of this thread's
// digit e.
template <bool COHERENT, bool WITH_TSTART, int ITEMS>
__device__ __forceinline__ void tile_offsets(SortSmem<ITEMS> &sm, const SortArgs &a,
                                             const PassInfo &P, const TileGeom &g,
                                             const uint32_t (&tcount)[2], const uint32_t *gc)
{
    // Counts are tile- and group-major, so each load instruction reads 32
    // consecutive digits; the loops are unrolled so the loads are in flight
    // together.
    const int kg = g.k / kTilesPerGroup;
    const uint32_t *segg = gc + (size_t)g.seg * a.gps * kRadixMax;
    const uint32_t *segt = a.tile_cnt + (size_t)g.seg * a.tps * kRadixMax;
    uint32_t total[2] = {0u, 0u}, excl[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        if (e < P.dpt && d < P.ndig) {
            for (int g0 = 0; g0 < a.gps; g0 += 8) {
                uint32_t c[8];
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    c[q] = g0 + q < a.gps
                               ? load_u32<COHERENT>(segg + (size_t)(g0 + q) * kRadixMax + d)
                               : 0u;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    total[e] += c[q];
                    if (g0 + q < kg)
                        excl[e] += c[q];
                }
            }
            const int t0 = kg * kTilesPerGroup;
            for (int q0 = 0; q0 < kTilesPerGroup; q0 += 16) {
                uint32_t c[16];
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    c[q] = t0 + q0 + q < g.k
                               ? load_u32<COHERENT>(segt + (size_t)(t0 + q0 + q) * kRadixMax + d)
                               : 0u;
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    excl[e] += c[q];
            }
        }
    }

    // The start of each digit in the segment is a scan over the threads'
    // digits; with WITH_TSTART the same scan also gives the tile-local start
    // (low half).
    const uint32_t seg_base = (uint32_t)(g.seg * a.L);
    uint32_t dbase, tstart = 0;
    if constexpr (WITH_TSTART) {
        const unsigned long long both = block_exclusive_scan64(
            ((unsigned long long)(total[0] + total[1]) << 32) | (tcount[0] + tcount[1]),
            (unsigned long long *)sm.warp2);
        tstart = (uint32_t)both;
        dbase = (uint32_t)(both >> 32);
    } else {
        dbase = block_exclusive_scan(total[0] + total[1], sm.warp, nullptr);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        if (e < P.dpt && d < P.ndig) {
            if constexpr (WITH_TSTART) {
                sm.tstart[d] = tstart;
                tstart += tcount[e];
            }
            sm.gbase[d] = seg_base + dbase + excl[e] - sm.tstart[d];
            dbase += total[e];
        }
    }
    __syncthreads();
}

// The item as the pass writes it: the last pass turns the segment-relative
// key back into the row.
__device__ __forceinline__ unsigned long long out_item(unsigned long long x, const SortArgs &a,
                                                      const PassInfo &P, int seg)
{
    return P.last ? x + ((unsigned long long)(uint32_t)a.off[seg] << 32) : x;
}

// Writes a staged tile (sm.items, ordered by digit) to its sorted positions,
// once every tile of the pass has published its counts.
template <bool COHERENT, int ITEMS>
__device__ __forceinline__ void place_staged_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                                  const PassInfo &P, unsigned long long *dst,
                                                  const TileGeom &g,
                                                  const uint32_t (&tcount)[2],
                                                  const uint32_t *gc)
{
    tile_offsets<COHERENT, false>(sm, a, P, g, tcount, gc);
    for (int p = threadIdx.x; p < g.count; p += kSortThreads) {
        const unsigned long long x = sm.items[p];
        dst[(uint32_t)(sm.gbase[digit_of(x, P)] + (uint32_t)p)] = out_item(x, a, P, g.seg);
    }
    __syncthreads(); // shared memory free for the next tile
}

// Count phase of the one-launch sort when tiles outnumber the resident
// blocks (a block cannot keep its tiles across the barrier): stages the tile
// and writes it back ordered by digit into its own region of `ordered`, so
// that the place phase need not rank it again. `ordered` may be `src` itself
// (the tile region is read before it is written, by this block alone).
template <int ITEMS>
__device__ __forceinline__ void count_order_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                                 const void *src, const PassInfo &P, int tile,
                                                 uint32_t *gc, unsigned long long *ordered)
{
    const TileGeom g = tile_geom(a, tile, SortSmem<ITEMS>::kTile);
    uint32_t tcount[2];
    stage_tile<true>(sm, a, src, P, tile, g, P.first, gc, tcount);
    for (int q = threadIdx.x; q < g.count; q += kSortThreads)
        ordered[g.begin + q] = sm.items[q];
    __syncthreads(); // shared memory free for the next tile
}

// Place phase for a tile that count_order_tile left ordered by digit: each
// run of one digit goes to that digit's positions.
template <int ITEMS>
__device__ __forceinline__ void place_ordered_tile(SortSmem<ITEMS> &sm, const SortArgs &a,
                                                   const PassInfo &P,
                                                   const unsigned long long *ordered,
                                                   unsigned long long *dst, int tile,
                                                   const uint32_t *gc)
{
    const TileGeom g = tile_geom(a, tile, SortSmem<ITEMS>::kTile);
    uint32_t tcount[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int d = my_digit(P, e);
        if (e < P.dpt && d < P.ndig)
            tcount[e] = __ldcg(a.tile_cnt + (size_t)tile * kRadixMax + d);
    }
    tile_offsets<true, true>(sm, a, P, g, tcount, gc);
    for (int q = threadIdx.x; q < g.count; q += kSortThreads) {
        const unsigned long long x = __ldcg(ordered + g.begin + q);
        dst[(uint32_t)(sm.gbase[digit_of(x, P)] + (uint32_t)q)] = out_item(x, a, P, g.seg);
    }
    __syncthreads(); // shared memory free for the next tile
}

// ----------------------------------------------- one launch per phase

template <int ITEMS>
__global__ void __launch_bounds__(kSortThreads) radix_count(SortArgs a, int pass)
{
    __shared__ SortSmem<ITEMS> sm;
    const PassInfo P = pass_info(a, pass);
    const void *src = P.first ? nullptr : out_buffer(a, pass - 1);
    count_tile(sm, a, src, P, blockIdx.x, a.group_cnt + (size_t)pass * a.ngroups * kRadixMax);
}

template <int ITEMS>
__global__ void __launch_bounds__(kSortThreads) radix_scatter(SortArgs a, int pass)
{
    __shared__ SortSmem<ITEMS> sm;
    const PassInfo P = pass_info(a, pass);
    const void *src = P.first ? nullptr : out_buffer(a, pass - 1);
    const TileGeom g = tile_geom(a, blockIdx.x, SortSmem<ITEMS>::kTile);
    uint32_t tcount[2];
    // (the count phase has already published the counts and checked the keys)
    stage_tile<false>(sm, a, src, P, blockIdx.x, g, false, nullptr, tcount);
    place_staged_tile<false>(sm, a, P, out_buffer(a, pass), g, tcount,
                             a.group_cnt + (size_t)pass * a.ngroups * kRadixMax);
}

// ------------------------------------------------ one cooperative launch

// Grid-wide barrier among co-resident blocks on one arrival counter that only
// grows: barrier k of the launch is passed once the counter reaches
// k * gridDim.x. Thread 0 of each block arrives with one acquire-release add
// and, unless it was the last to arrive, polls the counter with acquire loads
// (at most spin_limit polls; giving up raises ENGRAM_DEVERR_SORT_TIMEOUT and
// returns false). The block's other threads wait at __syncthreads, which
// orders their later reads after thread 0's acquire. The counter is zero at
// launch. A block reaches barrier k only after passing barrier k - 1, so a
// block that passes barrier k sees every block's writes before it.
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

// Four blocks per SM keep 592 tiles resident on a 148-SM B200.
template <int ITEMS> __global__ void __launch_bounds__(kSortThreads, 4) radix_sort_coop(SortArgs a)
{
    __shared__ SortSmem<ITEMS> sm;
    constexpr int TILE = SortSmem<ITEMS>::kTile;
    unsigned gen = 0;
    if (a.ntiles <= (int)gridDim.x) {
        // One tile per block: rank it once and keep it staged in shared
        // memory, ordered by digit, across the barrier; then place it.
        const int tile = blockIdx.x;
        const bool has = tile < a.ntiles;
        const TileGeom g = tile_geom(a, has ? tile : 0, TILE);
        for (int pass = 0; pass < a.passes; ++pass) {
            const PassInfo P = pass_info(a, pass);
            const void *src = P.first ? nullptr : out_buffer(a, pass - 1);
            uint32_t *gc = a.group_cnt + (size_t)pass * a.ngroups * kRadixMax;
            uint32_t tcount[2] = {0u, 0u};
            if (has)
                stage_tile<true>(sm, a, src, P, tile, g, P.first, gc, tcount);
            if (!grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
                return;
            if (has)
                place_staged_tile<true>(sm, a, P, out_buffer(a, pass), g, tcount, gc);
            if (!P.last && !grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
                return;
        }
        return;
    }
    // More tiles than resident blocks: each tile is ranked once, in the count
    // phase, and left ordered by digit in `ordered` (the pass's own input from
    // the second pass on; on the first, whose input is idx, the buffer the
    // pass does not write), from where the place phase moves it.
    for (int pass = 0; pass < a.passes; ++pass) {
        const PassInfo P = pass_info(a, pass);
        unsigned long long *dst = out_buffer(a, pass);
        unsigned long long *src = P.first ? nullptr : out_buffer(a, pass - 1);
        unsigned long long *ordered = P.first ? (dst == a.a ? a.b : a.a) : src;
        uint32_t *gc = a.group_cnt + (size_t)pass * a.ngroups * kRadixMax;
        for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x)
            count_order_tile(sm, a, src, P, tile, gc, ordered);
        if (!grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
            return;
        for (int tile = blockIdx.x; tile < a.ntiles; tile += gridDim.x)
            place_ordered_tile(sm, a, P, ordered, dst, tile, gc);
        if (!P.last && !grid_barrier(a.barrier, gen, sm.flag, a.spin_limit))
            return;
    }
}

} // namespace bwd
} // namespace engram
