// owner.cuh -- routing of lookups to the ranks that own their table rows
// (engram page, Qwen3_8_FlashNextOwnerShardedEmbedding: rank r owns rows
// [r * rows_per_owner, (r + 1) * rows_per_owner); a requesting rank groups
// its row IDs by owner before the first All-to-All, and the values come back
// in the same grouping).
//
// A stable counting sort of the n lookups by owner o = row / rows_per_owner
// (at most 256 owners), in three launches over 2048-lookup tiles:
//   owner_count    per-tile owner counts (shared-memory adds, one per
//                  distinct owner in a warp);
//   owner_scan     one block: per owner, the exclusive sum over tiles, and
//                  the owners' totals and starts;
//   owner_scatter  every tile ranks its lookups stably (peers of equal owner
//                  in a warp by __match_any_sync, per-warp running counts in
//                  shared memory, warps in order) and writes, for grouped
//                  position p of lookup i:
//                    send_rows[p] = row - o * rows_per_owner  (owner-local row)
//                    src_pos[p]   = i        (where the values go back to)
//                    dst_pos[i]   = p
// so lookups of one owner keep their original order. A row outside
// [0, owners * rows_per_owner) is routed to the last owner with local row -1,
// which that owner's lookup rejects, and raises ENGRAM_DEVERR_ROW_RANGE here.
// In the fixed-capacity layout (the pages' _fixed_capacity_all_to_all: every
// owner's segment padded to one capacity agreed ahead of time, so the
// exchanges have static sizes and need no counts on the host), owner o's
// lookups go to positions o * cap + rank, the rest of the segment is padding
// (-1), and lookups past the capacity are dropped (dst_pos -1) with
// ENGRAM_DEVERR_CAPACITY.
#pragma once

#include "common.cuh"

namespace engram {
namespace owner {

constexpr int kThreads = 256;
constexpr int kItems = 8;
constexpr int kTile = kThreads * kItems;  // 2048 lookups per tile
constexpr int kWarps = kThreads / 32;
constexpr int kMaxOwners = 256;

struct OwnerArgs {
    const int32_t *rows;
    int64_t n;
    int64_t rows_per_owner;
    int32_t owners, ntiles;
    uint32_t *tile_cnt;   // [ntiles][owners]
    uint32_t *tile_off;   // [ntiles][owners] exclusive starts (owner start + earlier tiles)
    int32_t *counts;      // [owners]
    int32_t *send_rows, *src_pos, *dst_pos;
    int64_t cap;          // > 0: fixed-capacity segments [owners][cap]; 0: compact
};

__device__ __forceinline__ int owner_of(int32_t row, const OwnerArgs &a, bool &bad)
{
    const int64_t o = row < 0 ? -1 : (int64_t)row / a.rows_per_owner;
    bad = o < 0 || o >= a.owners;
    return bad ? a.owners - 1 : (int)o;
}

// The owner-local row of `row` (owner o), or -1 for a row no owner holds.
__device__ __forceinline__ int32_t local_row(int32_t row, int o, const OwnerArgs &a)
{
    const int64_t l = (int64_t)row - (int64_t)o * a.rows_per_owner;
    return l >= 0 && l < a.rows_per_owner ? (int32_t)l : -1;
}

__global__ void __launch_bounds__(kThreads) owner_count(const OwnerArgs a)
{
    __shared__ uint32_t cnt[kMaxOwners];
    const int tid = threadIdx.x, lane = tid & 31;
    for (int o = tid; o < a.owners; o += kThreads)
        cnt[o] = 0;
    __syncthreads();
    const int64_t base = (int64_t)blockIdx.x * kTile;
    bool bad_any = false;
#pragma unroll
    for (int r = 0; r < kItems; ++r) {
        const int64_t i = base + r * kThreads + tid;
        const bool valid = i < a.n;
        bool bad = false;
        const int o = valid ? owner_of(__ldg(a.rows + i), a, bad) : -1 - lane;
        bad_any |= valid && bad;
        const uint32_t peers = __match_any_sync(kFull, o);
        if (valid && lane == __ffs(peers) - 1)
            atomicAdd(&cnt[o], (uint32_t)__popc(peers));
    }
    if (bad_any)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    __syncthreads();
    for (int o = tid; o < a.owners; o += kThreads)
        a.tile_cnt[(size_t)blockIdx.x * a.owners + o] = cnt[o];
}

// One block: thread o walks the tiles in order for owner o.
__global__ void __launch_bounds__(kThreads) owner_scan(const OwnerArgs a)
{
    __shared__ uint32_t total[kMaxOwners];
    const int o = threadIdx.x;
    uint32_t run = 0;
    if (o < a.owners) {
        for (int t0 = 0; t0 < a.ntiles; t0 += 8) {
            uint32_t c[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                c[q] = t0 + q < a.ntiles ? a.tile_cnt[(size_t)(t0 + q) * a.owners + o] : 0u;
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (t0 + q < a.ntiles) {
                    a.tile_off[(size_t)(t0 + q) * a.owners + o] = run;
                    run += c[q];
                }
        }
        total[o] = run;
        if (a.cap > 0 && (int64_t)run > a.cap)
            raise_device_error(ENGRAM_DEVERR_CAPACITY);
        a.counts[o] = (int32_t)(a.cap > 0 ? min64(run, a.cap) : run);
    }
    __syncthreads();
    if (o < a.owners) {
        // owner o's segment starts after the earlier owners' lookups, or at
        // o * cap in the fixed-capacity layout
        int64_t start = 0;
        if (a.cap > 0)
            start = (int64_t)o * a.cap;
        else
            for (int q = 0; q < o; ++q)
                start += total[q];
        for (int t = 0; t < a.ntiles; ++t)
            a.tile_off[(size_t)t * a.owners + o] += (uint32_t)start;
    }
}

__global__ void __launch_bounds__(kThreads) owner_scatter(const OwnerArgs a)
{
    __shared__ uint32_t wcnt[kWarps][kMaxOwners];
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    for (int k = tid; k < kWarps * a.owners; k += kThreads)
        wcnt[k / a.owners][k % a.owners] = 0;
    __syncthreads();
    // warp w ranks lookups [w * 256, (w + 1) * 256) of the tile, 32 at a time
    const int64_t wbase = (int64_t)blockIdx.x * kTile + (int64_t)wid * (32 * kItems);
    const uint32_t lt = (1u << lane) - 1u;
    int32_t row[kItems];
    int own[kItems];
    uint32_t rank[kItems];
#pragma unroll
    for (int r = 0; r < kItems; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        const bool valid = i < a.n;
        bool bad = false;
        row[r] = valid ? __ldg(a.rows + i) : 0;
        own[r] = valid ? owner_of(row[r], a, bad) : -1 - lane;
        const uint32_t peers = __match_any_sync(kFull, own[r]);
        const int leader = __ffs(peers) - 1;
        uint32_t before = 0;
        if (valid && lane == leader) {
            before = wcnt[wid][own[r]];
            wcnt[wid][own[r]] = before + __popc(peers);
        }
        before = __shfl_sync(kFull, before, leader);
        rank[r] = before + __popc(peers & lt);
        __syncwarp();
    }
    __syncthreads();
    // per owner: exclusive offsets of the warps within the tile
    for (int o = tid; o < a.owners; o += kThreads) {
        uint32_t run = a.tile_off[(size_t)blockIdx.x * a.owners + o];
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const uint32_t c = wcnt[w][o];
            wcnt[w][o] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kItems; ++r) {
        const int64_t i = wbase + r * 32 + lane;
        if (i < a.n) {
            const uint32_t p = wcnt[wid][own[r]] + rank[r];
            if (a.cap > 0 && (int64_t)p - (int64_t)own[r] * a.cap >= a.cap) {
                a.dst_pos[i] = -1; // past the owner's capacity: dropped (flagged by the scan)
                continue;
            }
            a.send_rows[p] = local_row(row[r], own[r], a);
            a.src_pos[p] = (int32_t)i;
            a.dst_pos[i] = (int32_t)p;
        }
    }
    // fixed-capacity layout: the unused slots of every owner's segment are
    // padding (row -1, position -1), which the lookups and the backward skip
    if (a.cap > 0) {
        const int64_t slots = a.cap * a.owners;
        for (int64_t k = (int64_t)blockIdx.x * kThreads + tid; k < slots;
             k += (int64_t)gridDim.x * kThreads) {
            const int o = (int)(k / a.cap);
            if (k - (int64_t)o * a.cap >= a.counts[o]) {
                a.send_rows[k] = -1;
                a.src_pos[k] = -1;
            }
        }
    }
}

} // namespace owner
} // namespace engram
