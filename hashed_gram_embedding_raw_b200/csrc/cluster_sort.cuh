// cluster_sort.cuh -- the backward's sort by head done on chip, one
// thread-block cluster per head.
//
// The sort by head (radix_sort.cuh) orders each head's T lookups on its own:
// segment h holds lookup t * H + h at position t and is sorted by
// row - offset[h]. When a segment fits the shared memory of one cluster of
// kClusterCtas blocks (T <= kClusterCtas * kClusterCap: 65,536 lookups, the
// page's 16 x 4,096-token batch), the whole segment stays on chip for every
// pass: block c of the cluster holds positions [c * cap, (c + 1) * cap) of
// the segment, and each pass
//   1. ranks the block's items stably by digit (per-warp digit counters,
//      peers by one ballot per digit bit) and counts each digit in the block;
//   2. after a cluster barrier, reads every block's digit counts through
//      distributed shared memory: digit d of block c starts at
//        sum over digits d' < d of their totals in the segment
//        + the counts of d in blocks before c;
//   3. stores each item straight into the shared memory of the block that
//      owns its position in the next order (st.shared::cluster), then a
//      second cluster barrier makes those stores visible.
// Pass 0 reads the int32 row indices from global memory (keyed relative to
// the head's first row); after the last pass each block writes its positions
// to the output buffer with the head's offset added back, the same items the
// grid-wide sort leaves. No global memory is touched between passes and no
// block waits on anything outside its cluster. Every pass is a stable
// counting sort of the digit, so equal rows keep ascending lookup order.
#pragma once

#include "radix_sort.cuh"

namespace engram {
namespace bwd {

constexpr int kClusterCtas = 8;                             // blocks per cluster (portable)
constexpr int kClusterThreads = 512;
constexpr int kClusterWarps = kClusterThreads / 32;
constexpr int kClusterItems = 16;                           // items per thread
constexpr int kClusterCap = kClusterThreads * kClusterItems; // positions per block: 8,192
constexpr int kClusterMaxSegment = kClusterCtas * kClusterCap;

// Dynamic shared memory of a block: two item buffers, per-warp digit
// counters, the block's digit counts (read by the other blocks), digit starts
// and scan scratch.
struct ClusterSmem {
    unsigned long long buf[2][kClusterCap];
    uint32_t whist[kClusterWarps][kRadixMax];
    uint32_t ccount[kRadixMax];
    uint32_t start[kRadixMax];
    uint32_t warp[32];
};

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of the cluster; shared-memory accesses (local and remote) before
// it are visible to those after it.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-window address of the same object in block `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(const void *local, uint32_t rank)
{
    uint32_t remote;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                 : "=r"(remote)
                 : "r"((uint32_t)__cvta_generic_to_shared(local)), "r"(rank));
    return remote;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ void st_cluster_u64(uint32_t addr, unsigned long long v)
{
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}

// One cluster per segment (a.S clusters of kClusterCtas blocks). Writes the
// sorted segment to a.a; a.L <= kClusterMaxSegment.
__global__ void __launch_bounds__(kClusterThreads, 1) cluster_sort_kernel(SortArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    ClusterSmem &sm = *reinterpret_cast<ClusterSmem *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const uint32_t crank = cluster_ctarank();
    const int seg = blockIdx.x / kClusterCtas;
    const int cap = (int)((a.L + kClusterCtas - 1) / kClusterCtas);
    const int lo = (int)crank * cap;
    const int cnt = max(0, min(cap, (int)a.L - lo)); // this block's positions
    const uint32_t lt = lanemask_lt();
    const int wbase = wid * (32 * kClusterItems);

    int cur = 0; // buffer holding this pass's input
    bool bad = false;
    for (int pass = 0; pass < a.passes; ++pass) {
        const PassInfo P = pass_info(a, pass);
        // items of this block, in position order: item i = wbase + r * 32 + lane
        uint64_t it[kClusterItems];
#pragma unroll
        for (int r = 0; r < kClusterItems; ++r) {
            const int i = wbase + r * 32 + lane;
            if (i < cnt) {
                if (P.first) {
                    it[r] = first_item(a, seg, (int64_t)(lo + i) * a.S + seg, bad);
                } else {
                    it[r] = sm.buf[cur][i];
                }
            } else {
                it[r] = 0;
            }
        }
        for (int k = tid; k < (kClusterWarps << P.bits); k += kClusterThreads)
            sm.whist[k >> P.bits][k & (P.ndig - 1)] = 0;
        __syncthreads();
        // 1. stable rank inside the warp, per-warp digit counts
        uint32_t rank[kClusterItems];
#pragma unroll
        for (int r = 0; r < kClusterItems; ++r) {
            const bool valid = wbase + r * 32 + lane < cnt;
            const uint32_t dg = digit_of(it[r], P);
            const uint32_t peers = digit_peers(dg, valid, P.bits);
            const int leader = valid ? __ffs(peers) - 1 : lane;
            uint32_t c = 0;
            if (valid && lane == leader) {
                c = sm.whist[wid][dg];
                sm.whist[wid][dg] = c + __popc(peers);
            }
            c = __shfl_sync(kFull, c, leader);
            rank[r] = c + __popc(peers & lt);
            __syncwarp();
        }
        __syncthreads();
        // per digit: the warps' exclusive offsets in the block, and the
        // block's count, published for the other blocks
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int d = tid * P.dpt + e;
            if (e < P.dpt && d < P.ndig) {
                uint32_t run = 0;
#pragma unroll
                for (int w = 0; w < kClusterWarps; ++w) {
                    const uint32_t c = sm.whist[w][d];
                    sm.whist[w][d] = run;
                    run += c;
                }
                sm.ccount[d] = run;
            }
        }
        cluster_sync_all(); // every block's counts are out
        // 2. the digit's start in the segment for this block
        uint32_t tot[2] = {0u, 0u}, before[2] = {0u, 0u};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int d = tid * P.dpt + e;
            if (e < P.dpt && d < P.ndig) {
                uint32_t c[kClusterCtas];
#pragma unroll
                for (int q = 0; q < kClusterCtas; ++q)
                    c[q] = ld_cluster_u32(map_rank(&sm.ccount[d], (uint32_t)q));
#pragma unroll
                for (int q = 0; q < kClusterCtas; ++q) {
                    tot[e] += c[q];
                    if (q < (int)crank)
                        before[e] += c[q];
                }
            }
        }
        uint32_t dbase = block_exclusive_scan<false>(tot[0] + tot[1], sm.warp, nullptr);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int d = tid * P.dpt + e;
            if (e < P.dpt && d < P.ndig) {
                sm.start[d] = dbase + before[e];
                dbase += tot[e];
            }
        }
        __syncthreads();
        // 3. each item to its position's block, into the other buffer
        const int nxt = cur ^ 1;
#pragma unroll
        for (int r = 0; r < kClusterItems; ++r) {
            if (wbase + r * 32 + lane < cnt) {
                const uint32_t dg = digit_of(it[r], P);
                const uint32_t p = sm.start[dg] + sm.whist[wid][dg] + rank[r];
                const uint32_t dst = p / (uint32_t)cap;
                const uint32_t off = p - dst * (uint32_t)cap;
                st_cluster_u64(map_rank(&sm.buf[nxt][off], dst), it[r]);
            }
        }
        cluster_sync_all(); // the next order is complete in every block
        cur = nxt;
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
    // the sorted segment, with the head's first row added back to the key
    const unsigned long long offhi = (unsigned long long)(uint32_t)a.off[seg] << 32;
    unsigned long long *out = a.a + (int64_t)seg * a.L + lo;
    for (int i = tid; i < cnt; i += kClusterThreads)
        out[i] = sm.buf[cur][i] + offhi;
}

} // namespace bwd
} // namespace engram
