// engram.cu -- C ABI of the Engram N-gram Embedding library (include/engram.h).
//
// Host side: argument checks (ENGRAM_EINVAL before anything is launched),
// launch planning (grid sized to the resident warps of the current device,
// work cut into balanced contiguous per-warp ranges), workspace layout of the
// backward, and the device error word. All arithmetic runs in the kernels of
// hash_gather.cuh and backward.cuh.
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <tuple>

#include "engram.h"

#include "backward.cuh"
#include "common.cuh"
#include "hash_gather.cuh"
#include "ple_conv.cuh"
#include "ple_conv_bwd.cuh"
#include "ple_conv_cls.cuh"
#include "optim.cuh"
#include "owner.cuh"
#include "norm.cuh"

using namespace engram;

namespace {

std::atomic<uint64_t> g_launches{0};

int after_launch()
{
    if (cudaGetLastError() != cudaSuccess)
        return ENGRAM_ECUDA;
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return ENGRAM_OK;
}

#define ENGRAM_TRY(expr)                                                                   \
    do {                                                                                   \
        const int rc_ = (expr);                                                            \
        if (rc_ != ENGRAM_OK)                                                              \
            return rc_;                                                                    \
    } while (0)

int device_sms(int *sms)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return ENGRAM_ECUDA;
    static std::atomic<int> cache[128];
    if (dev >= 0 && dev < 128) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *sms = c;
            return ENGRAM_OK;
        }
    }
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
        return ENGRAM_ECUDA;
    if (dev >= 0 && dev < 128)
        cache[dev].store(v, std::memory_order_relaxed);
    *sms = v;
    return ENGRAM_OK;
}

// Resident warps of `fn` on the current device with the given block shape.
template <typename F>
int resident_warps(F fn, int threads, size_t smem, int64_t *warps)
{
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return ENGRAM_ECUDA;
    ENGRAM_TRY(device_sms(&sms));
    static std::mutex mu;
    static std::map<std::tuple<const void *, int, int, size_t>, int> cache;
    const auto key = std::make_tuple((const void *)fn, dev, threads, smem);
    int nb = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end())
            nb = it->second;
    }
    if (nb == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem) != cudaSuccess)
            return ENGRAM_ECUDA;
        if (nb < 1)
            nb = 1;
        std::lock_guard<std::mutex> lock(mu);
        cache[key] = nb;
    }
    *warps = (int64_t)sms * nb * (threads / 32);
    return ENGRAM_OK;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int elem_bytes(int32_t dtype)
{
    switch (dtype) {
    case ENGRAM_F32:
        return 4;
    case ENGRAM_BF16:
    case ENGRAM_F16:
        return 2;
    default:
        return 0;
    }
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int make_hash_args(const engram_params_t *p, HashArgs *a)
{
    if (p == nullptr)
        return ENGRAM_EINVAL;
    const int N = p->ngram_size, K = p->heads_per_ngram;
    if (N < 2 || N > ENGRAM_MAX_NGRAM || K < 1 || K > ENGRAM_MAX_HEADS ||
        (N - 1) * K > ENGRAM_MAX_HEADS)
        return ENGRAM_EINVAL;
    if (p->table_rows < 1 || p->table_rows > (int64_t(1) << 31) || p->dim < 1)
        return ENGRAM_EINVAL;
    std::memset(a, 0, sizeof(*a));
    a->N = N;
    a->K = K;
    a->H = (N - 1) * K;
    a->eos = p->eos_id;
    a->fill = p->fill_id;
    for (int k = 0; k < N; ++k)
        a->mult[k] = p->multipliers[k];
    for (int h = 0; h < a->H; ++h) {
        const int64_t v = p->vocab_sizes[h], o = p->offsets[h];
        if (v < 1 || o < 0 || o > p->table_rows - v)
            return ENGRAM_EINVAL;
        a->p[h] = (uint64_t)v;
        a->magic[h] = UINT64_MAX / (uint64_t)v;
        a->off[h] = (int32_t)o;
    }
    return ENGRAM_OK;
}

// ---------------------------------------------------------------- forward

int launch_hash(const HashArgs &a, const int32_t *ids, const int32_t *cu, int32_t nseq,
                int64_t T, int32_t *out_idx, cudaStream_t stream)
{
    const size_t smem = (size_t)(kHashThreads / 32) * 32 * (a.H + 1) * sizeof(int32_t);
    const bool page_shape = a.N == 3 && a.K == 8;
    auto fn = page_shape ? hash_kernel<3, 8> : hash_kernel<0, 0>;
    int64_t res = 0;
    ENGRAM_TRY(resident_warps(fn, kHashThreads, smem, &res));
    const int64_t nwarps = std::min<int64_t>(res, ceil_div(T, 32));
    const int64_t blocks = ceil_div(nwarps, kHashThreads / 32);
    fn<<<(unsigned)blocks, kHashThreads, smem, stream>>>(a, ids, cu, nseq, T, nwarps, out_idx);
    return after_launch();
}

// slice == nullptr: the whole stream; else only the slice's nlog tokens.
int launch_hash_gather(const HashArgs &a, const int32_t *ids, const int32_t *cu, int32_t nseq,
                       int64_t T, const void *table, int V, int32_t *out_idx, void *out,
                       cudaStream_t stream, const SliceMap *slice = nullptr, int64_t nlog = 0)
{
    const size_t smem = (size_t)(kHashThreads / 32) * 32 * (a.H + 1) * sizeof(int32_t);
    const bool page_shape = a.N == 3 && a.K == 8;
    const bool mapped = slice != nullptr;
    auto fn = mapped ? hash_gather_kernel<0, 0, 0, true> : hash_gather_kernel<0, 0, 0, false>;
    if (page_shape && V == 20)
        fn = mapped ? hash_gather_kernel<3, 8, 20, true> : hash_gather_kernel<3, 8, 20, false>;
    else if (page_shape && V == 40)
        fn = mapped ? hash_gather_kernel<3, 8, 40, true> : hash_gather_kernel<3, 8, 40, false>;
    int64_t res = 0;
    ENGRAM_TRY(resident_warps(fn, kHashThreads, smem, &res));
    const int64_t units = mapped ? nlog : T;
    const int64_t nwarps = std::max<int64_t>(1, std::min<int64_t>(res, ceil_div(units, 8)));
    const int64_t blocks = ceil_div(nwarps, kHashThreads / 32);
    const SliceMap m = mapped ? *slice : SliceMap{0, 0, 1};
    fn<<<(unsigned)blocks, kHashThreads, smem, stream>>>(a, ids, cu, nseq, T, nwarps,
                                                         (const uint4 *)table, V, out_idx,
                                                         (uint4 *)out, m, nlog);
    return after_launch();
}

// --------------------------------------------------------------- backward

// Workspace layout of the backward for n lookups: large enough for the sort
// of either form (one segment, or one per head) at any tile size.
struct BwdPlan {
    int wmax = 0, GF = 0, tiles_max = 0, groups_max = 0;
    int64_t rows = 0;
    size_t a = 0, b = 0, tile_cnt = 0, ctl = 0, ctl_bytes = 0, group_cnt = 0, barrier = 0;
    size_t wcount = 0, bcount = 0, pb = 0, pe = 0, meta = 0, total = 0;
};

int bwd_plan(int64_t n, int64_t rows, int32_t dim, BwdPlan *P)
{
    if (n < 0 || n > INT32_MAX || rows < 1 || rows > (int64_t(1) << 31) || dim < 8 ||
        dim % 8 != 0 || dim > 512)
        return ENGRAM_EINVAL;
    int sms = 0;
    ENGRAM_TRY(device_sms(&sms));
    P->rows = rows;
    // warps of seg_reduce: at most 32 per SM (its resident limit) and one per
    // 32 lookups, so the fp64 partials below shrink with small n
    P->wmax = (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)sms * 32, ceil_div(n, 32)));
    P->GF = (dim / 4 + 31) / 32;
    // the smallest tiles, plus one short tile per segment at most
    P->tiles_max = (int)(ceil_div(std::max<int64_t>(n, 1),
                                  (int64_t)bwd::kSortThreads * bwd::kSortItemsMin) +
                         bwd::kMaxSegments);
    P->groups_max = (int)(ceil_div(P->tiles_max, bwd::kTilesPerGroup) + bwd::kMaxSegments);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~size_t(255);
        return at;
    };
    const size_t nn = (size_t)std::max<int64_t>(n, 1);
    P->a = take(nn * 8);
    P->b = take(nn * 8);
    // per-tile digit counts (rewritten by every pass), and per-group digit
    // sums of every pass (accumulated with atomic adds, zeroed once per sort)
    P->tile_cnt = take((size_t)bwd::kRadixMax * P->tiles_max * 4);
    P->ctl = off;
    P->group_cnt = take((size_t)bwd::kMaxPasses * bwd::kRadixMax * P->groups_max * 4);
    P->barrier = take(sizeof(unsigned)); // grid-barrier counter of the one-launch sort
    P->ctl_bytes = off - P->ctl;
    P->wcount = take((size_t)P->wmax * 4);
    P->bcount = take((size_t)ceil_div(P->wmax, bwd::kSegWarps) * 4);
    P->pb = take((size_t)P->wmax * dim * 8);
    P->pe = take((size_t)P->wmax * dim * 8);
    P->meta = take((size_t)P->wmax * sizeof(bwd::SegMeta));
    P->total = off;
    return ENGRAM_OK;
}

int check_workspace(const BwdPlan &P, void *ws, size_t ws_bytes)
{
    if (ws == nullptr || ((uintptr_t)ws & 255u) != 0)
        return ENGRAM_EINVAL;
    if (ws_bytes < P.total)
        return ENGRAM_ENOSPC;
    return ENGRAM_OK;
}

// What one sort orders: S segments of L lookups; segment s holds keys
// off[s] .. off[s] + size[s] - 1 and is sorted by key - off[s].
struct SortShape {
    int S = 1;
    int64_t L = 0;
    int32_t off[bwd::kMaxSegments] = {};
    uint32_t size[bwd::kMaxSegments] = {};
    bool pad = false; // negative indices are absent lookups, keyed size[s]
};

int bit_width(uint64_t v) // bits needed for 0 .. v
{
    int b = 0;
    while (b < 64 && (v >> b) != 0)
        ++b;
    return b;
}

// The plain sort: one segment of all n lookups over the whole table; with
// `pad`, a negative index is an absent lookup that sorts after every row.
SortShape plain_shape(int64_t n, int64_t rows, bool pad)
{
    SortShape sh;
    sh.S = 1;
    sh.L = n;
    sh.off[0] = 0;
    sh.size[0] = (uint32_t)std::min<int64_t>(rows, UINT32_MAX);
    sh.pad = pad;
    return sh;
}

// The sort by head: lookup j = t * H + h of T tokens lies in head h's slice.
// Needs ascending, disjoint slices inside the table; otherwise the plain sort.
SortShape head_shape(const engram_params_t *p, int64_t T)
{
    const int H = (p->ngram_size - 1) * p->heads_per_ngram;
    bool ok = H >= 1 && H <= bwd::kMaxSegments;
    for (int h = 0; ok && h < H; ++h) {
        const int64_t o = p->offsets[h], v = p->vocab_sizes[h];
        ok = v >= 1 && o >= 0 && o + v <= p->table_rows && o <= INT32_MAX &&
             (h == 0 || o >= p->offsets[h - 1] + p->vocab_sizes[h - 1]);
    }
    if (!ok)
        return plain_shape(T * std::max(H, 1), p->table_rows, false);
    SortShape sh;
    sh.S = H;
    sh.L = T;
    for (int h = 0; h < H; ++h) {
        sh.off[h] = (int32_t)p->offsets[h];
        sh.size[h] = (uint32_t)p->vocab_sizes[h];
    }
    return sh;
}

template <int I> int sort_resident_blocks(int64_t *blocks)
{
    int64_t warps = 0;
    ENGRAM_TRY(resident_warps(bwd::radix_sort_coop<I>, bwd::kSortThreads, 0, &warps));
    *blocks = warps / (bwd::kSortThreads / 32);
    return ENGRAM_OK;
}

int64_t shape_tiles(const SortShape &sh, int items)
{
    return sh.S * std::max<int64_t>(1, ceil_div(sh.L, (int64_t)bwd::kSortThreads * items));
}

// Pairs per thread of the sort's tiles (4..8). Among the sizes that keep every
// tile resident at once (the one-launch sort then holds a block's items in
// registers across the grid barrier), take the one whose busiest SM holds the
// fewest pairs -- 512 tiles of 2048 on 148 SMs leave 68 SMs with four tiles
// and 80 with three; 592 tiles of 1792 give every SM four smaller ones. With
// none resident, the largest tiles.
int sort_items(const SortShape &sh, int sms, int *items)
{
    int64_t res[bwd::kSortItemsMax + 1] = {};
    ENGRAM_TRY(sort_resident_blocks<4>(&res[4]));
    ENGRAM_TRY(sort_resident_blocks<5>(&res[5]));
    ENGRAM_TRY(sort_resident_blocks<6>(&res[6]));
    ENGRAM_TRY(sort_resident_blocks<7>(&res[7]));
    ENGRAM_TRY(sort_resident_blocks<8>(&res[8]));
    int best = bwd::kSortItemsMax;
    int64_t best_load = INT64_MAX;
    for (int I = bwd::kSortItemsMax; I >= bwd::kSortItemsMin; --I) {
        const int64_t tiles = shape_tiles(sh, I);
        if (tiles > res[I])
            continue;
        const int64_t load = ceil_div(tiles, (int64_t)sms) * I;
        if (load < best_load) {
            best = I;
            best_load = load;
        }
    }
    *items = best;
    return ENGRAM_OK;
}

uint32_t barrier_spin_limit();

// Kernel arguments of a sort of `sh` on tiles of 256 * items pairs, inside
// the workspace laid out by P.
int sort_args(const int32_t *idx, const SortShape &sh, int items, const BwdPlan &P, char *ws,
              bwd::SortArgs *out)
{
    using namespace bwd;
    SortArgs &a = *out;
    std::memset(&a, 0, sizeof(a));
    int key_bits = 1; // the largest key: size - 1, or size for an absent lookup
    for (int s = 0; s < sh.S; ++s)
        key_bits = std::max(key_bits, bit_width((uint64_t)sh.size[s] - (sh.pad ? 0 : 1)));
    a.passes = (key_bits + kDigitBitsMax - 1) / kDigitBitsMax;
    if (a.passes > kMaxPasses)
        return ENGRAM_EINVAL;
    for (int q = 0; q < a.passes; ++q) // spread the bits evenly, wider digits first
        a.bits[q] = key_bits / a.passes + (q < key_bits % a.passes ? 1 : 0);
    const int64_t tile = (int64_t)kSortThreads * items;
    a.idx = idx;
    a.a = (unsigned long long *)(ws + P.a);
    a.b = (unsigned long long *)(ws + P.b);
    a.S = sh.S;
    a.L = sh.L;
    a.n = (int64_t)sh.S * sh.L;
    a.tps = (int)std::max<int64_t>(1, ceil_div(sh.L, tile));
    a.gps = (int)ceil_div(a.tps, kTilesPerGroup);
    a.ntiles = a.S * a.tps;
    a.ngroups = a.S * a.gps;
    if (a.ntiles > P.tiles_max || a.ngroups > P.groups_max)
        return ENGRAM_EINVAL;
    a.tile_cnt = (uint32_t *)(ws + P.tile_cnt);
    a.group_cnt = (uint32_t *)(ws + P.group_cnt);
    a.barrier = (unsigned *)(ws + P.barrier);
    a.spin_limit = barrier_spin_limit();
    for (int s = 0; s < sh.S; ++s) {
        a.off[s] = sh.off[s];
        a.size[s] = sh.size[s];
    }
    a.pad = sh.pad;
    return ENGRAM_OK;
}

// The one-launch sort at I pairs per thread; *launched is false where the
// device or the launch refuses a cooperative grid (nothing ran).
template <int I>
int launch_sort_coop(const int32_t *idx, const SortShape &sh, const BwdPlan &P, char *ws,
                     cudaStream_t stream, bool *launched)
{
    using namespace bwd;
    *launched = false;
    int dev = 0, coop = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
        return ENGRAM_OK;
    SortArgs args;
    ENGRAM_TRY(sort_args(idx, sh, I, P, ws, &args));
    // the grid is at most the co-resident blocks, which the launch itself checks
    int64_t res = 0;
    ENGRAM_TRY(resident_warps(radix_sort_coop<I>, kSortThreads, 0, &res));
    const int grid = (int)std::min<int64_t>(args.ntiles, res / (kSortThreads / 32));
    void *params[] = {&args};
    if (cudaLaunchCooperativeKernel((const void *)radix_sort_coop<I>, dim3(grid),
                                    dim3(kSortThreads), params, 0, stream) != cudaSuccess) {
        (void)cudaGetLastError();
        return ENGRAM_OK;
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    *launched = true;
    return ENGRAM_OK;
}

// ENGRAM_SORT_SEPARATE_LAUNCHES=1 in the environment (read once per process)
// makes the sort take its two-launches-per-pass form, the one devices without
// cooperative launch get, so that it can be checked on a device that has it.
bool sort_separate_launches()
{
    static const bool v = [] {
        const char *e = std::getenv("ENGRAM_SORT_SEPARATE_LAUNCHES");
        return e != nullptr && e[0] == '1';
    }();
    return v;
}

// Test hooks for the bounded waits: ENGRAM_TEST_BARRIER_SPIN=<polls> caps the
// sort's grid-barrier polls and ENGRAM_TEST_CROSS_WAIT_NS=<ns> the PLE tail
// kernel's waits on other warps (both read once per process). Small values
// make a wait run out in a test -- the call then ends with the matching
// ENGRAM_DEVERR_* bit set instead of the result; unset, the waits keep their
// normal bounds (about 0.3 s and 0.5 s).
uint64_t env_u64(const char *name, uint64_t fallback)
{
    const char *e = std::getenv(name);
    if (e == nullptr || e[0] == '\0')
        return fallback;
    char *end = nullptr;
    const unsigned long long v = std::strtoull(e, &end, 10);
    return (end != nullptr && *end == '\0') ? (uint64_t)v : fallback;
}

uint32_t barrier_spin_limit()
{
    static const uint32_t v = (uint32_t)std::min<uint64_t>(
        env_u64("ENGRAM_TEST_BARRIER_SPIN", bwd::kBarrierSpin), bwd::kBarrierSpin);
    return v;
}

uint64_t cross_wait_ns()
{
    static const uint64_t v =
        std::min<uint64_t>(env_u64("ENGRAM_TEST_CROSS_WAIT_NS", ple::kCopyWaitNs),
                           ple::kCopyWaitNs);
    return v;
}

// Sorts the pairs of `sh` into buffer a of the workspace: the grid-wide sort
// in one cooperative launch, else two launches per pass.
int launch_sort(const int32_t *idx, const SortShape &sh, const BwdPlan &P, char *ws,
                cudaStream_t stream)
{
    using namespace bwd;
    bool launched = false;
    if (cudaMemsetAsync(ws + P.ctl, 0, P.ctl_bytes, stream) != cudaSuccess)
        return ENGRAM_ECUDA;
    int items = 0;
    if (!sort_separate_launches()) {
        int sms = 0;
        ENGRAM_TRY(device_sms(&sms));
        ENGRAM_TRY(sort_items(sh, sms, &items));
    }
    switch (items) {
    case 0: break;
    case 4: ENGRAM_TRY(launch_sort_coop<4>(idx, sh, P, ws, stream, &launched)); break;
    case 5: ENGRAM_TRY(launch_sort_coop<5>(idx, sh, P, ws, stream, &launched)); break;
    case 6: ENGRAM_TRY(launch_sort_coop<6>(idx, sh, P, ws, stream, &launched)); break;
    case 7: ENGRAM_TRY(launch_sort_coop<7>(idx, sh, P, ws, stream, &launched)); break;
    case 8: ENGRAM_TRY(launch_sort_coop<8>(idx, sh, P, ws, stream, &launched)); break;
    default: return ENGRAM_EINVAL;
    }
    if (launched)
        return ENGRAM_OK;

    // Without a cooperative launch: two launches per pass, on the largest
    // tiles (2,048 pairs).
    constexpr int I = kSortItemsMax;
    SortArgs args;
    ENGRAM_TRY(sort_args(idx, sh, I, P, ws, &args));
    for (int pass = 0; pass < args.passes; ++pass) {
        radix_count<I><<<args.ntiles, kSortThreads, 0, stream>>>(args, pass);
        ENGRAM_TRY(after_launch());
        radix_scatter<I><<<args.ntiles, kSortThreads, 0, stream>>>(args, pass);
        ENGRAM_TRY(after_launch());
    }
    return ENGRAM_OK;
}

template <int DT, int GF, int RVT>
int launch_seg(const unsigned long long *items, int64_t n, const BwdPlan &P, const void *dout,
               int dim, int32_t *uniq, float *grads, int32_t *num_unique, char *ws,
               cudaStream_t stream)
{
    using namespace bwd;
    const int row_bytes = dim * (DT == ENGRAM_F32 ? 4 : 2);
    const int batch = std::max(1, std::min(kSegMaxBatch, kSegStageBytes / row_bytes));
    const int stage_bytes = batch * row_bytes;
    const size_t smem = (size_t)kSegWarps * kSegStages * (stage_bytes + kSegMaxBatch * 8);
    auto fn = seg_reduce<DT, GF, RVT>;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return ENGRAM_ECUDA;
    int64_t res = 0;
    ENGRAM_TRY(resident_warps(fn, kSegThreads, smem, &res));
    const int W = (int)std::max<int64_t>(
        1, std::min<int64_t>(std::min<int64_t>(res, P.wmax), ceil_div(n, 32)));
    const int blocks = (int)ceil_div(W, kSegWarps);
    auto *wcount = (uint32_t *)(ws + P.wcount);
    auto *bcount = (uint32_t *)(ws + P.bcount);
    auto *pb = (double *)(ws + P.pb);
    auto *pe = (double *)(ws + P.pe);
    auto *meta = (SegMeta *)(ws + P.meta);
    // an absent lookup's item has key table_rows: its run is no distinct row
    seg_count<<<blocks, kSegThreads, 0, stream>>>(items, n, W, (uint32_t)P.rows, wcount,
                                                  bcount);
    ENGRAM_TRY(after_launch());
    fn<<<blocks, kSegThreads, smem, stream>>>(items, n, W, wcount, bcount, dout, dim, batch,
                                              stage_bytes, uniq, grads, pb, pe, meta,
                                              num_unique);
    ENGRAM_TRY(after_launch());
    seg_fixup<GF><<<blocks, kSegThreads, 0, stream>>>(W, dim, pb, pe, meta, uniq, grads);
    return after_launch();
}

template <int DT>
int launch_seg_dt(const unsigned long long *items, int64_t n, const BwdPlan &P,
                  const void *dout, int dim, int32_t *uniq, float *grads, int32_t *num_unique,
                  char *ws, cudaStream_t stream)
{
    // the page's 160-wide rows get a compile-time row width
    constexpr int kRow160 = 160 * (DT == ENGRAM_F32 ? 4 : 2) / 16;
    if (dim == 160)
        return launch_seg<DT, 2, kRow160>(items, n, P, dout, dim, uniq, grads, num_unique, ws,
                                          stream);
    switch (P.GF) {
    case 1:
        return launch_seg<DT, 1, 0>(items, n, P, dout, dim, uniq, grads, num_unique, ws, stream);
    case 2:
        return launch_seg<DT, 2, 0>(items, n, P, dout, dim, uniq, grads, num_unique, ws, stream);
    default:
        return launch_seg<DT, 4, 0>(items, n, P, dout, dim, uniq, grads, num_unique, ws, stream);
    }
}

int launch_reduce(int64_t n, int32_t dim, const void *dout, int32_t dtype, int32_t *uniq,
                  float *grads, int32_t *num_unique, const BwdPlan &P, char *ws,
                  cudaStream_t stream)
{
    if (n == 0) {
        if (cudaMemsetAsync(num_unique, 0, sizeof(int32_t), stream) != cudaSuccess)
            return ENGRAM_ECUDA;
        return ENGRAM_OK;
    }
    const auto *items = (const unsigned long long *)(ws + P.a); // the sort's last pass wrote a
    switch (dtype) {
    case ENGRAM_F32:
        return launch_seg_dt<ENGRAM_F32>(items, n, P, dout, dim, uniq, grads, num_unique, ws,
                                         stream);
    case ENGRAM_BF16:
        return launch_seg_dt<ENGRAM_BF16>(items, n, P, dout, dim, uniq, grads, num_unique, ws,
                                          stream);
    default:
        return launch_seg_dt<ENGRAM_F16>(items, n, P, dout, dim, uniq, grads, num_unique, ws,
                                         stream);
    }
}

int check_reduce_args(int64_t n, const void *dout, int32_t dtype, int32_t *uniq, float *grads,
                      int32_t *num_unique)
{
    if (elem_bytes(dtype) == 0 || num_unique == nullptr)
        return ENGRAM_EINVAL;
    if (n > 0 && (dout == nullptr || uniq == nullptr || grads == nullptr ||
                  !aligned16(dout) || !aligned16(grads)))
        return ENGRAM_EINVAL;
    return ENGRAM_OK;
}

// The hash's lookups: n = T * H, lookup t * H + h in head h's slice.
int heads_args(const engram_params_t *params, int64_t T, int64_t *n)
{
    HashArgs a;
    ENGRAM_TRY(make_hash_args(params, &a));
    if (T < 0 || T * a.H > INT32_MAX)
        return ENGRAM_EINVAL;
    *n = T * a.H;
    return ENGRAM_OK;
}

} // namespace

// =============================================================== C ABI

extern "C" {

int engram_hash(const engram_params_t *params, const int32_t *ids, const int32_t *cu_seqlens,
                int32_t nseq, int64_t T, int32_t *out_idx, engram_stream_t stream)
{
    HashArgs a;
    ENGRAM_TRY(make_hash_args(params, &a));
    if (T < 0 || T > INT32_MAX || (cu_seqlens != nullptr && nseq < 1))
        return ENGRAM_EINVAL;
    if (T == 0)
        return ENGRAM_OK;
    if (ids == nullptr || out_idx == nullptr)
        return ENGRAM_EINVAL;
    return launch_hash(a, ids, cu_seqlens, nseq, T, out_idx, (cudaStream_t)stream);
}

int engram_gather(const void *table, int32_t dtype, int64_t table_rows, int32_t dim,
                  const int32_t *idx, int64_t n, void *out, engram_stream_t stream)
{
    const int eb = elem_bytes(dtype);
    if (eb == 0 || dim < 1 || ((int64_t)dim * eb) % 16 != 0 || table_rows < 1 || n < 0)
        return ENGRAM_EINVAL;
    if (n == 0)
        return ENGRAM_OK;
    if (table == nullptr || idx == nullptr || out == nullptr || !aligned16(table) ||
        !aligned16(out))
        return ENGRAM_EINVAL;
    const int V = (int)((int64_t)dim * eb / 16);
    auto fn = V == 20 ? gather_kernel<20> : V == 40 ? gather_kernel<40> : gather_kernel<0>;
    int64_t res = 0;
    ENGRAM_TRY(resident_warps(fn, kHashThreads, 0, &res));
    const int64_t nwarps = std::min<int64_t>(res, ceil_div(n, 32));
    const int64_t blocks = ceil_div(nwarps, kHashThreads / 32);
    fn<<<(unsigned)blocks, kHashThreads, 0, (cudaStream_t)stream>>>(
        (const uint4 *)table, table_rows, V, idx, n, nwarps, (uint4 *)out);
    return after_launch();
}

int engram_hash_gather(const engram_params_t *params, const int32_t *ids,
                       const int32_t *cu_seqlens, int32_t nseq, int64_t T, const void *table,
                       int32_t dtype, int32_t *out_idx, void *out, engram_stream_t stream)
{
    HashArgs a;
    ENGRAM_TRY(make_hash_args(params, &a));
    const int eb = elem_bytes(dtype);
    if (eb == 0 || ((int64_t)params->dim * eb) % 16 != 0)
        return ENGRAM_EINVAL;
    if (T < 0 || T > INT32_MAX || (cu_seqlens != nullptr && nseq < 1))
        return ENGRAM_EINVAL;
    if (T == 0)
        return ENGRAM_OK;
    if (ids == nullptr || table == nullptr || out == nullptr || !aligned16(table) ||
        !aligned16(out))
        return ENGRAM_EINVAL;
    const int V = (int)((int64_t)params->dim * eb / 16);
    return launch_hash_gather(a, ids, cu_seqlens, nseq, T, table, V, out_idx, out,
                              (cudaStream_t)stream);
}

int engram_hash_gather_slice(const engram_params_t *params, const int32_t *ids,
                             const int32_t *cu_seqlens, int32_t nseq, int64_t T, int64_t row_len,
                             int64_t start, int64_t end, const void *table, int32_t dtype,
                             int32_t *out_idx, void *out, engram_stream_t stream)
{
    HashArgs a;
    ENGRAM_TRY(make_hash_args(params, &a));
    const int eb = elem_bytes(dtype);
    if (eb == 0 || ((int64_t)params->dim * eb) % 16 != 0)
        return ENGRAM_EINVAL;
    if (T < 0 || T > INT32_MAX || (cu_seqlens != nullptr && nseq < 1))
        return ENGRAM_EINVAL;
    const int64_t row = row_len == 0 ? T : row_len;
    if (row < 0 || (row > 0 && T % row != 0) || start < 0 || end < start || end > row)
        return ENGRAM_EINVAL;
    const int64_t len = end - start;
    if (T == 0 || len == 0)
        return ENGRAM_OK;
    if (ids == nullptr || table == nullptr || out == nullptr || !aligned16(table) ||
        !aligned16(out))
        return ENGRAM_EINVAL;
    const int V = (int)((int64_t)params->dim * eb / 16);
    const SliceMap m{row, start, len};
    return launch_hash_gather(a, ids, cu_seqlens, nseq, T, table, V, out_idx, out,
                              (cudaStream_t)stream, &m, (T / row) * len);
}

int engram_backward_workspace_size(int64_t n, int64_t table_rows, int32_t dim, size_t *bytes)
{
    if (bytes == nullptr)
        return ENGRAM_EINVAL;
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, table_rows, dim, &P));
    *bytes = P.total;
    return ENGRAM_OK;
}

int engram_backward_sort(const int32_t *idx, int64_t n, int64_t table_rows, int32_t dim,
                         void *workspace, size_t workspace_bytes, engram_stream_t stream)
{
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, table_rows, dim, &P));
    ENGRAM_TRY(check_workspace(P, workspace, workspace_bytes));
    if (n == 0)
        return ENGRAM_OK;
    if (idx == nullptr)
        return ENGRAM_EINVAL;
    return launch_sort(idx, plain_shape(n, table_rows, true), P, (char *)workspace,
                       (cudaStream_t)stream);
}

int engram_backward_reduce(int64_t n, int64_t table_rows, int32_t dim, const void *dout,
                           int32_t dtype, int32_t *uniq_rows, float *row_grads,
                           int32_t *num_unique, void *workspace, size_t workspace_bytes,
                           engram_stream_t stream)
{
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, table_rows, dim, &P));
    ENGRAM_TRY(check_workspace(P, workspace, workspace_bytes));
    ENGRAM_TRY(check_reduce_args(n, dout, dtype, uniq_rows, row_grads, num_unique));
    return launch_reduce(n, dim, dout, dtype, uniq_rows, row_grads, num_unique, P,
                         (char *)workspace, (cudaStream_t)stream);
}

int engram_backward(const int32_t *idx, int64_t n, int64_t table_rows, int32_t dim,
                    const void *dout, int32_t dtype, int32_t *uniq_rows, float *row_grads,
                    int32_t *num_unique, void *workspace, size_t workspace_bytes,
                    engram_stream_t stream)
{
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, table_rows, dim, &P));
    ENGRAM_TRY(check_workspace(P, workspace, workspace_bytes));
    ENGRAM_TRY(check_reduce_args(n, dout, dtype, uniq_rows, row_grads, num_unique));
    if (n > 0 && idx == nullptr)
        return ENGRAM_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    if (n > 0)
        ENGRAM_TRY(launch_sort(idx, plain_shape(n, table_rows, true), P, (char *)workspace, s));
    return launch_reduce(n, dim, dout, dtype, uniq_rows, row_grads, num_unique, P,
                         (char *)workspace, s);
}

int engram_backward_sort_heads(const engram_params_t *params, const int32_t *idx, int64_t T,
                               void *workspace, size_t workspace_bytes, engram_stream_t stream)
{
    int64_t n = 0;
    ENGRAM_TRY(heads_args(params, T, &n));
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, params->table_rows, params->dim, &P));
    ENGRAM_TRY(check_workspace(P, workspace, workspace_bytes));
    if (n == 0)
        return ENGRAM_OK;
    if (idx == nullptr)
        return ENGRAM_EINVAL;
    return launch_sort(idx, head_shape(params, T), P, (char *)workspace, (cudaStream_t)stream);
}

int engram_backward_heads(const engram_params_t *params, const int32_t *idx, int64_t T,
                          const void *dout, int32_t dtype, int32_t *uniq_rows, float *row_grads,
                          int32_t *num_unique, void *workspace, size_t workspace_bytes,
                          engram_stream_t stream)
{
    int64_t n = 0;
    ENGRAM_TRY(heads_args(params, T, &n));
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, params->table_rows, params->dim, &P));
    ENGRAM_TRY(check_workspace(P, workspace, workspace_bytes));
    ENGRAM_TRY(check_reduce_args(n, dout, dtype, uniq_rows, row_grads, num_unique));
    if (n > 0 && idx == nullptr)
        return ENGRAM_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    if (n > 0)
        ENGRAM_TRY(launch_sort(idx, head_shape(params, T), P, (char *)workspace, s));
    return launch_reduce(n, params->dim, dout, dtype, uniq_rows, row_grads, num_unique, P,
                         (char *)workspace, s);
}

} // extern "C"

// ------------------------------------------------- allocation-free backward

namespace {

// Scratch of engram_backward_noalloc: one array per device, loaded with the
// library and held until the process exits. In host code this name only
// stands for the array; its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ENGRAM_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device, looked up on the
// first call per device (with that device current) and cached.
int noalloc_scratch(char **ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128)
        return ENGRAM_ECUDA;
    static std::mutex mu;
    static char *cache[128] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev] == nullptr) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return ENGRAM_ECUDA;
        cache[dev] = (char *)p;
    }
    *ptr = cache[dev];
    return ENGRAM_OK;
}

} // namespace

extern "C" {

int engram_backward_noalloc(const int32_t *idx, int64_t n, int64_t table_rows, int32_t dim,
                            const void *dout, int32_t dtype, int32_t *uniq_rows,
                            float *row_grads, int32_t *num_unique, engram_stream_t stream)
{
    BwdPlan P;
    ENGRAM_TRY(bwd_plan(n, table_rows, dim, &P));
    if (P.total > ENGRAM_NOALLOC_SCRATCH_BYTES)
        return ENGRAM_ENOSPC;
    ENGRAM_TRY(check_reduce_args(n, dout, dtype, uniq_rows, row_grads, num_unique));
    if (n > 0 && idx == nullptr)
        return ENGRAM_EINVAL;
    char *ws = nullptr;
    ENGRAM_TRY(noalloc_scratch(&ws));
    cudaStream_t s = (cudaStream_t)stream;
    // launch_sort clears the sort's control block in the array on every call
    if (n > 0)
        ENGRAM_TRY(launch_sort(idx, plain_shape(n, table_rows, true), P, ws, s));
    return launch_reduce(n, dim, dout, dtype, uniq_rows, row_grads, num_unique, P, ws, s);
}

int engram_get_device_error(uint32_t *flags, engram_stream_t stream)
{
    if (flags == nullptr)
        return ENGRAM_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    void *addr = nullptr;
    unsigned int v = 0;
    if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess)
        return ENGRAM_ECUDA;
    if (cudaMemcpyAsync(&v, addr, sizeof(v), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return ENGRAM_ECUDA;
    if (cudaMemsetAsync(addr, 0, sizeof(v), s) != cudaSuccess)
        return ENGRAM_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return ENGRAM_ECUDA;
    *flags = v;
    return ENGRAM_OK;
}

const char *engram_status_string(int status)
{
    switch (status) {
    case ENGRAM_OK:
        return "ENGRAM_OK: success";
    case ENGRAM_EINVAL:
        return "ENGRAM_EINVAL: invalid argument (nothing launched)";
    case ENGRAM_ENOSPC:
        return "ENGRAM_ENOSPC: workspace too small (nothing launched)";
    case ENGRAM_ECUDA:
        return "ENGRAM_ECUDA: CUDA launch or runtime call failed";
    default:
        return "unknown engram status";
    }
}

int engram_abi_version(void) { return ENGRAM_ABI_VERSION; }

size_t engram_params_size(void) { return sizeof(engram_params_t); }

uint64_t engram_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int64_t engram_host_floor_mod(int64_t a, int64_t m, int *status)
{
    if (m < 1 || m > (int64_t)UINT32_MAX) {
        if (status)
            *status = ENGRAM_EINVAL;
        return 0;
    }
    if (status)
        *status = ENGRAM_OK;
    return floor_mod(a, (uint64_t)m, UINT64_MAX / (uint64_t)m);
}

} // extern "C"

// ------------------------------------------------------ PLE layer tail

namespace {

struct ConvPlan {
    ple::ConvArgs a;
    size_t smem = 0;
    int grid = 0, threads = 0, chan = 4;
    bool cls = false;  // kernel width <= 4, one residue class per block
};

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t x = (uintptr_t)a, y = (uintptr_t)b;
    return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

// Checks the shape (host only) and sizes the block: G / 4 threads of 4
// channels (G / 8 of 8 for branches wider than 2,560) and the private rings
// of the normalised history. conv_grid adds the grid: one block per (branch,
// range), sms / branches blocks per branch.
int conv_plan(const engram_conv_params_t *p, int32_t dtype, int32_t out_dtype, int64_t T,
              ConvPlan *P)
{
    if (p == nullptr)
        return ENGRAM_EINVAL;
    const int eb = elem_bytes(dtype);
    if (eb == 0 || elem_bytes(out_dtype) == 0 || elem_bytes(p->weight_dtype) == 0 ||
        (out_dtype != dtype && out_dtype != ENGRAM_F32))
        return ENGRAM_EINVAL;
    const int C = p->channels, G = p->group_size, K = p->kernel_size, d = p->dilation;
    if (C < 1 || G < 8 || C % G != 0 || G % 8 != 0 || G / 8 > ple::kWideThreads)
        return ENGRAM_EINVAL;
    if (K < 1 || K > ple::kMaxTaps || d < 1 || d > 4096 || p->reserved != 0)
        return ENGRAM_EINVAL;
    if (!std::isfinite(p->eps) || p->eps < 0.f || (p->flags & ~7u) != 0)
        return ENGRAM_EINVAL;
    if (T < 0 || T > INT32_MAX)
        return ENGRAM_EINVAL;
    const int halo = (K - 1) * d;
    const int chan = G / 4 <= ple::kNarrowThreads ? 4 : 8;  // channels per thread
    const int nth = G / chan;
    const int norm_slots = halo + ple::kRows;
    // kernel widths up to 4 on branches up to 2,560 channels (4 per thread):
    // one residue class per block, batches of 8 rows in shared memory, any
    // dilation; otherwise the chunked kernel, whose private history rings
    // must fit shared memory
    const int pitch_reg = (G * eb + 127) / 128 * 128;  // bytes per buffered row
    const int cls_bufs = (int)std::min<size_t>(
        ple::kClsMaxBufs,
        (ple::kSmemLimit - ple::kClsDataOffset) / ((size_t)ple::kClsRows * pitch_reg));
    P->cls = K <= ple::kClsTaps && G / 4 <= 32 * ple::kClsMaxConvWarps && cls_bufs >= 2;
    if (!P->cls && ple::smem_bytes(norm_slots, nth, chan) > ple::kSmemLimit)
        return ENGRAM_EINVAL;
    ple::ConvArgs &a = P->a;
    std::memset(&a, 0, sizeof(a));
    a.T = T;
    a.C = C;
    a.G = G;
    a.nth = nth;
    a.wdtype = p->weight_dtype;
    a.eps = p->eps;
    a.groups = C / G;
    a.inv_G = 1.f / (float)G;
    a.K = K;
    a.dil = d;
    a.halo = halo;
    a.norm_slots = norm_slots;
    a.flags = p->flags;
    a.cross_wait_ns = cross_wait_ns();
    P->chan = chan;
    P->threads = (nth + 31) / 32 * 32;
    P->smem = ple::smem_bytes(norm_slots, nth, chan);
    if (P->cls) {
        P->chan = 4;
        a.nth = G / P->chan;
        a.reg_bufs = cls_bufs;
        a.pitch = pitch_reg;
        P->threads = 32 * ((a.nth + 31) / 32 + ple::kClsStatWarps);
        P->smem = ple::cls_smem_bytes(cls_bufs, pitch_reg);
    }
    return ENGRAM_OK;
}

// Grid of a checked plan on the current device (T > 0).
int conv_grid(ConvPlan *P)
{
    int sms = 0;
    ENGRAM_TRY(device_sms(&sms));
    const int groups = P->a.C / P->a.G;
    if (P->cls) {
        // branches x residues x chunks, about one block per SM
        const int classes = (int)std::max<int64_t>(1, std::min<int64_t>(P->a.dil, P->a.T));
        const int64_t rows = std::max<int64_t>(1, ceil_div(P->a.T, P->a.dil));
        int64_t chunks = std::max<int64_t>(1, sms / ((int64_t)groups * classes));
        chunks = std::min<int64_t>(chunks, std::max<int64_t>(1, ceil_div(rows, 32)));
        const int64_t grid = (int64_t)groups * classes * chunks;
        if (grid > INT32_MAX)
            return ENGRAM_EINVAL;
        P->a.classes = classes;
        P->a.bpg = (int32_t)chunks;
        P->grid = (int)grid;
        return ENGRAM_OK;
    }
    int64_t bpg = std::max(1, sms / groups);
    bpg = std::min<int64_t>(bpg, std::max<int64_t>(1, ceil_div(P->a.T, 64)));
    if ((int64_t)groups * bpg > INT32_MAX)
        return ENGRAM_EINVAL;
    P->a.bpg = (int32_t)bpg;
    P->grid = (int)(groups * bpg);
    return ENGRAM_OK;
}

// Raises the dynamic shared-memory limit of `fn` to the block maximum, once
// per device (the limit only gates launches; it reserves nothing).
template <typename F>
int allow_smem(F fn)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return ENGRAM_ECUDA;
    static std::mutex mu;
    static std::set<std::pair<const void *, int>> done;
    const auto key = std::make_pair((const void *)fn, dev);
    std::lock_guard<std::mutex> lock(mu);
    if (done.count(key) == 0) {
        if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ple::kSmemLimit) != cudaSuccess)
            return ENGRAM_ECUDA;
        done.insert(key);
    }
    return ENGRAM_OK;
}

// Kernel widths up to 4 on branches up to 2,560 channels (the page's shape):
// the residue-class kernel. Otherwise the chunked kernel, 4 channels per
// thread up to 2,560 channels, 8 beyond.
template <typename XT, typename OT>
int launch_conv_t(const ConvPlan &P, cudaStream_t s)
{
    if (P.cls) {
        auto fc = P.a.inv_out != nullptr ? ple::short_conv_cls_kernel<XT, OT, 4, true>
                                         : ple::short_conv_cls_kernel<XT, OT, 4, false>;
        ENGRAM_TRY(allow_smem(fc));
        fc<<<P.grid, P.threads, P.smem, s>>>(P.a);
        return after_launch();
    }
    const bool save = P.a.inv_out != nullptr;
    auto fn = P.chan == 8 ? (save ? ple::short_conv_kernel<XT, OT, 0, 8, true>
                                  : ple::short_conv_kernel<XT, OT, 0, 8, false>)
                          : (save ? ple::short_conv_kernel<XT, OT, 0, 4, true>
                                  : ple::short_conv_kernel<XT, OT, 0, 4, false>);
    ENGRAM_TRY(allow_smem(fn));
    fn<<<P.grid, P.threads, P.smem, s>>>(P.a);
    return after_launch();
}

int launch_conv(ConvPlan &P, int32_t dtype, int32_t out_dtype, cudaStream_t s)
{
    ENGRAM_TRY(conv_grid(&P));
    const bool f32_out = out_dtype == ENGRAM_F32;
    switch (dtype) {
    case ENGRAM_F32:
        return launch_conv_t<float, float>(P, s);
    case ENGRAM_BF16:
        return f32_out ? launch_conv_t<__nv_bfloat16, float>(P, s)
                       : launch_conv_t<__nv_bfloat16, __nv_bfloat16>(P, s);
    default:
        return f32_out ? launch_conv_t<__half, float>(P, s) : launch_conv_t<__half, __half>(P, s);
    }
}

} // namespace

extern "C" {

int engram_ple_short_conv_save(const engram_conv_params_t *params, const void *x,
                               int32_t dtype, const int32_t *cu_seqlens, int32_t nseq, int64_t T,
                               const void *norm_weight, const void *conv_weight,
                               const void *conv_bias, void *out, int32_t out_dtype,
                               float *inv_rms, engram_stream_t stream)
{
    ConvPlan P;
    ENGRAM_TRY(conv_plan(params, dtype, out_dtype, T, &P));
    if (cu_seqlens != nullptr && nseq < 1)
        return ENGRAM_EINVAL;
    if (inv_rms != nullptr && !(params->flags & ENGRAM_CONV_NORM))
        return ENGRAM_EINVAL;
    if (T == 0)
        return ENGRAM_OK;
    if (x == nullptr || out == nullptr || conv_weight == nullptr || !aligned16(x) ||
        !aligned16(out))
        return ENGRAM_EINVAL;
    const size_t n = (size_t)T * params->channels;
    if (overlaps(x, n * elem_bytes(dtype), out, n * elem_bytes(out_dtype)))
        return ENGRAM_EINVAL;
    if (inv_rms != nullptr) {
        const size_t ni = (size_t)T * (params->channels / params->group_size) * sizeof(float);
        if (((uintptr_t)inv_rms & 3) != 0 || overlaps(inv_rms, ni, x, n * elem_bytes(dtype)) ||
            overlaps(inv_rms, ni, out, n * elem_bytes(out_dtype)))
            return ENGRAM_EINVAL;
    }
    P.a.x = x;
    P.a.out = out;
    P.a.cu = cu_seqlens;
    P.a.nseq = cu_seqlens != nullptr ? nseq : 1;
    P.a.norm_w = norm_weight;
    P.a.conv_w = conv_weight;
    P.a.bias = conv_bias;
    P.a.inv_out = inv_rms;
    return launch_conv(P, dtype, out_dtype, (cudaStream_t)stream);
}

int engram_ple_short_conv(const engram_conv_params_t *params, const void *x, int32_t dtype,
                          const int32_t *cu_seqlens, int32_t nseq, int64_t T,
                          const void *norm_weight, const void *conv_weight,
                          const void *conv_bias, void *out, int32_t out_dtype,
                          engram_stream_t stream)
{
    return engram_ple_short_conv_save(params, x, dtype, cu_seqlens, nseq, T, norm_weight,
                                      conv_weight, conv_bias, out, out_dtype, nullptr, stream);
}

int engram_grouped_rms_norm(const void *x, int32_t dtype, int64_t rows, int32_t channels,
                            int32_t group_size, const void *weight, int32_t weight_dtype,
                            float eps, void *out, int32_t out_dtype, engram_stream_t stream)
{
    engram_conv_params_t p;
    std::memset(&p, 0, sizeof(p));
    p.channels = channels;
    p.group_size = group_size;
    p.kernel_size = 1;
    p.dilation = 1;
    p.eps = eps;
    p.flags = ENGRAM_CONV_NORM;
    p.weight_dtype = weight_dtype;
    ConvPlan P;
    ENGRAM_TRY(conv_plan(&p, dtype, out_dtype, rows, &P));
    if (rows == 0)
        return ENGRAM_OK;
    if (x == nullptr || out == nullptr || !aligned16(x) || !aligned16(out))
        return ENGRAM_EINVAL;
    // in place is allowed: a block writes a row only after reading it, and no
    // other block reads that row
    const size_t n = (size_t)rows * channels;
    if (out != x && overlaps(x, n * elem_bytes(dtype), out, n * elem_bytes(out_dtype)))
        return ENGRAM_EINVAL;
    if (out == x && out_dtype != dtype)
        return ENGRAM_EINVAL;
    const int eb = elem_bytes(dtype);
    const int nvec = group_size * eb / 16;  // 16-byte vectors per group slice
    if (nvec <= 32 * norm::kMaxVec) {
        // the streaming kernel: a warp per group slice, scales in shared memory
        int sms = 0;
        ENGRAM_TRY(device_sms(&sms));
        const int groups = channels / group_size;
        int64_t bpg = std::max<int64_t>(1, ceil_div((int64_t)sms * 4, groups));
        bpg = std::min<int64_t>(bpg, std::max<int64_t>(1, ceil_div(rows, 16)));
        if ((int64_t)groups * bpg > INT32_MAX)
            return ENGRAM_EINVAL;
        norm::NormArgs na;
        na.x = x;
        na.out = out;
        na.w = weight;
        na.wdtype = weight_dtype;
        na.rows = rows;
        na.C = channels;
        na.G = group_size;
        na.bpg = (int32_t)bpg;
        na.eps = eps;
        na.inv_G = 1.f / (float)group_size;
        const int need = (nvec + 31) / 32;
        const size_t smem = (size_t)group_size * sizeof(float);
        const unsigned grid = (unsigned)(groups * bpg);
        cudaStream_t st = (cudaStream_t)stream;
        auto go = [&](auto fn) {
            ENGRAM_TRY(allow_smem(fn));
            fn<<<grid, norm::kThreads, smem, st>>>(na);
            return after_launch();
        };
        auto pick = [&](auto xt, auto ot) {
            using XT = decltype(xt);
            using OT = decltype(ot);
            if (need <= 1)
                return go(norm::norm_kernel<XT, OT, 1>);
            if (need <= 2)
                return go(norm::norm_kernel<XT, OT, 2>);
            if (need <= 4)
                return go(norm::norm_kernel<XT, OT, 4>);
            if (need <= 8)
                return go(norm::norm_kernel<XT, OT, 8>);
            if (need <= 10)
                return go(norm::norm_kernel<XT, OT, 10>);
            return go(norm::norm_kernel<XT, OT, 16>);
        };
        const bool f32_out = out_dtype == ENGRAM_F32;
        switch (dtype) {
        case ENGRAM_F32:
            return pick(float(), float());
        case ENGRAM_BF16:
            return f32_out ? pick(__nv_bfloat16(), float())
                           : pick(__nv_bfloat16(), __nv_bfloat16());
        default:
            return f32_out ? pick(__half(), float()) : pick(__half(), __half());
        }
    }
    P.a.x = x;
    P.a.out = out;
    P.a.nseq = 1;
    P.a.norm_w = weight;
    return launch_conv(P, dtype, out_dtype, (cudaStream_t)stream);
}

} // extern "C"

// ------------------------------------------------- PLE layer tail backward

namespace {

struct ConvBwdPlan {
    ple::ConvBwdArgs a;
    size_t smem = 0, ws = 0;
    int grid = 0, threads = 0, npart = 0;
    int32_t dtype = 0, grad_dtype = 0;
};

// Checks the shape (host only) and sizes the launch: a branch slice of G
// channels on 1, 2 or 4 blocks of a cluster (at most 1,280 channels each, 640
// with 4; 2 per thread; every block but the last a multiple of 8 channels so
// that every row copy starts and ends on 16 bytes), the fewest blocks whose
// rings of row slots leave a batch in flight ahead, the rings as deep as
// shared memory allows with two blocks per multiprocessor (one, with deeper
// rings, when two leave no batch ahead), and one block per (branch,
// residue, chunk) with chunks chosen so that one wave of clusters covers the
// device.
int conv_bwd_plan(const engram_conv_params_t *p, int32_t dtype, int32_t grad_dtype, int64_t T,
                  ConvBwdPlan *P)
{
    if (p == nullptr)
        return ENGRAM_EINVAL;
    const int ex = elem_bytes(dtype), eg = elem_bytes(grad_dtype);
    if (ex == 0 || eg == 0 || elem_bytes(p->weight_dtype) == 0)
        return ENGRAM_EINVAL;
    const int C = p->channels, G = p->group_size, K = p->kernel_size, d = p->dilation;
    if (C < 1 || G < 8 || C % G != 0 || G % 8 != 0 || G > ple::kBwdMaxChannels)
        return ENGRAM_EINVAL;
    if (K < 1 || K > ple::kBwdTaps || d < 1 || d > 4096 || p->reserved != 0)
        return ENGRAM_EINVAL;
    if (!std::isfinite(p->eps) || p->eps < 0.f || (p->flags & ~7u) != 0)
        return ENGRAM_EINVAL;
    if (T < 0 || T > INT32_MAX)
        return ENGRAM_EINVAL;
    int csize = 0, gca = 0, pitch_x = 0, pitch_g = 0, pitch_u = 0, ahead = 0;
    for (int cs = 1; cs <= ple::kBwdMaxCluster && ahead < 1; cs *= 2) {
        gca = (int)ceil_div(G, 8 * cs) * 8;
        const int threads = (gca / ple::kBwdCh + 31) / 32 * 32;
        if (gca > ple::kBwdBlockChannels || cs * (threads / 32) > ple::kBwdCols ||
            G - (cs - 1) * gca < 8)
            continue;
        pitch_x = (gca * ex + 127) / 128 * 128;
        pitch_g = (gca * eg + 127) / 128 * 128;
        pitch_u = gca * (int)sizeof(float);
        auto ahead_for = [&](size_t budget) {
            const int most = std::min(ple::kBwdMaxSlots / ple::kBwdRows - 3, ple::kBwdBars - 2);
            int n = 0;
            while (n < most && ple::bwd_smem_bytes(n + 1, pitch_x, pitch_g, pitch_u) <= budget)
                ++n;
            return n;
        };
        ahead = ahead_for(ple::kBwdTwoBlockSmem);
        if (ahead < 1)
            ahead = ahead_for(ple::kSmemLimit);
        csize = cs;
    }
    if (ahead < 1)
        return ENGRAM_EINVAL;
    ple::ConvBwdArgs &a = P->a;
    std::memset(&a, 0, sizeof(a));
    a.T = T;
    a.C = C;
    a.G = G;
    a.gca = gca;
    a.dil = d;
    a.K = K;
    a.wdtype = p->weight_dtype;
    a.eps = p->eps;
    a.groups = C / G;
    a.inv_G = 1.f / (float)G;
    a.flags = p->flags;
    a.ahead = ahead;
    a.nbx = ahead + 3;
    a.nbg = ahead + 2;
    a.pitch_x = pitch_x;
    a.pitch_g = pitch_g;
    a.pitch_u = pitch_u;
    a.csize = csize;
    P->smem = ple::bwd_smem_bytes(ahead, pitch_x, pitch_g, pitch_u);
    P->threads = (gca / ple::kBwdCh + 31) / 32 * 32;
    P->dtype = dtype;
    P->grad_dtype = grad_dtype;
    return ENGRAM_OK;
}

template <typename XT, typename GT>
int conv_bwd_clusters_t(const ConvBwdPlan &P, int *clusters)
{
    auto fn = P.a.gca == ple::kBwdBlockChannels ? ple::short_conv_bwd_kernel<XT, GT, true>
                                                : ple::short_conv_bwd_kernel<XT, GT, false>;
    ENGRAM_TRY(allow_smem(fn));
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)P.a.csize);
    cfg.blockDim = dim3((unsigned)P.threads);
    cfg.dynamicSmemBytes = P.smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P.a.csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(clusters, fn, &cfg) != cudaSuccess)
        return ENGRAM_ECUDA;
    return ENGRAM_OK;
}

template <typename XT>
int conv_bwd_clusters_x(const ConvBwdPlan &P, int *clusters)
{
    switch (P.grad_dtype) {
    case ENGRAM_F32:
        return conv_bwd_clusters_t<XT, float>(P, clusters);
    case ENGRAM_BF16:
        return conv_bwd_clusters_t<XT, __nv_bfloat16>(P, clusters);
    default:
        return conv_bwd_clusters_t<XT, __half>(P, clusters);
    }
}

// Clusters of a checked plan that are resident at once on the current
// device, asked once per (device, element types, cluster size, shared memory).
int conv_bwd_clusters(const ConvBwdPlan &P, int *clusters)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return ENGRAM_ECUDA;
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int, size_t, int>, int> known;
    const auto key = std::make_tuple(dev, (int)P.dtype, (int)P.grad_dtype, P.a.csize, P.smem,
                                     P.threads);
    {
        std::lock_guard<std::mutex> lock(mu);
        auto it = known.find(key);
        if (it != known.end()) {
            *clusters = it->second;
            return ENGRAM_OK;
        }
    }
    int n = 0;
    switch (P.dtype) {
    case ENGRAM_F32:
        ENGRAM_TRY(conv_bwd_clusters_x<float>(P, &n));
        break;
    case ENGRAM_BF16:
        ENGRAM_TRY(conv_bwd_clusters_x<__nv_bfloat16>(P, &n));
        break;
    default:
        ENGRAM_TRY(conv_bwd_clusters_x<__half>(P, &n));
        break;
    }
    if (n < 1)
        return ENGRAM_ECUDA;
    std::lock_guard<std::mutex> lock(mu);
    known[key] = n;
    *clusters = n;
    return ENGRAM_OK;
}

// Grid and workspace of a checked plan on the current device.
int conv_bwd_grid(ConvBwdPlan *P)
{
    ple::ConvBwdArgs &a = P->a;
    int clusters = 0;
    ENGRAM_TRY(conv_bwd_clusters(*P, &clusters));
    const int groups = a.C / a.G;
    const int classes = (int)std::max<int64_t>(1, std::min<int64_t>(a.dil, a.T));
    const int64_t rows = std::max<int64_t>(1, ceil_div(a.T, a.dil));  // rows of residue 0
    int64_t chunks = std::max<int64_t>(1, clusters / ((int64_t)groups * classes));
    chunks = std::min<int64_t>(chunks, std::max<int64_t>(1, ceil_div(rows, 16)));
    const int64_t grid = (int64_t)groups * classes * chunks * a.csize;
    if (grid > INT32_MAX)
        return ENGRAM_EINVAL;
    a.chunks = (int32_t)chunks;
    a.classes = classes;
    P->grid = (int)grid;
    P->npart = (int)(classes * chunks);
    P->ws = (size_t)P->npart * ple::kBwdQuantities * (size_t)a.C * sizeof(float);
    return ENGRAM_OK;
}

template <typename XT, typename GT>
int launch_conv_bwd_t(const ConvBwdPlan &P, cudaStream_t s)
{
    auto fn = P.a.gca == ple::kBwdBlockChannels ? ple::short_conv_bwd_kernel<XT, GT, true>
                                                : ple::short_conv_bwd_kernel<XT, GT, false>;
    ENGRAM_TRY(allow_smem(fn));
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)P.grid);
    cfg.blockDim = dim3((unsigned)P.threads);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P.a.csize;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, P.a) != cudaSuccess)
        return ENGRAM_ECUDA;
    return after_launch();
}

template <typename XT>
int launch_conv_bwd_x(const ConvBwdPlan &P, int32_t grad_dtype, cudaStream_t s)
{
    switch (grad_dtype) {
    case ENGRAM_F32:
        return launch_conv_bwd_t<XT, float>(P, s);
    case ENGRAM_BF16:
        return launch_conv_bwd_t<XT, __nv_bfloat16>(P, s);
    default:
        return launch_conv_bwd_t<XT, __half>(P, s);
    }
}

} // namespace

extern "C" {

int engram_ple_short_conv_backward_workspace_size(const engram_conv_params_t *params, int64_t T,
                                                  size_t *bytes)
{
    if (bytes == nullptr)
        return ENGRAM_EINVAL;
    ConvBwdPlan P;
    ENGRAM_TRY(conv_bwd_plan(params, ENGRAM_BF16, ENGRAM_BF16, T, &P));
    ENGRAM_TRY(conv_bwd_grid(&P));
    *bytes = P.ws;
    return ENGRAM_OK;
}

int engram_ple_short_conv_backward_saved(
    const engram_conv_params_t *params, const void *x, int32_t dtype, const int32_t *cu_seqlens,
    int32_t nseq, int64_t T, const void *norm_weight, const void *conv_weight,
    const void *conv_bias, const float *inv_rms, const void *dout, int32_t grad_dtype, void *dx,
    float *dnorm_weight, float *dconv_weight, float *dconv_bias, void *workspace,
    size_t workspace_bytes, engram_stream_t stream)
{
    ConvBwdPlan P;
    ENGRAM_TRY(conv_bwd_plan(params, dtype, grad_dtype, T, &P));
    if (cu_seqlens != nullptr && nseq < 1)
        return ENGRAM_EINVAL;
    if (inv_rms != nullptr &&
        (!(params->flags & ENGRAM_CONV_NORM) || ((uintptr_t)inv_rms & 3) != 0))
        return ENGRAM_EINVAL;
    P.a.inv_in = inv_rms;
    if (conv_weight == nullptr || dconv_weight == nullptr)
        return ENGRAM_EINVAL;
    const int C = params->channels, K = params->kernel_size;
    cudaStream_t s = (cudaStream_t)stream;
    if (T > 0) {
        if (x == nullptr || dout == nullptr || dx == nullptr || !aligned16(x) ||
            !aligned16(dout) || !aligned16(dx))
            return ENGRAM_EINVAL;
        const size_t n = (size_t)T * C;
        const size_t nx = n * elem_bytes(dtype), ng = n * elem_bytes(grad_dtype);
        if (overlaps(dx, ng, x, nx) || overlaps(dx, ng, dout, ng))
            return ENGRAM_EINVAL;
        if (workspace == nullptr || !aligned16(workspace))
            return ENGRAM_EINVAL;
        ENGRAM_TRY(conv_bwd_grid(&P));
        if (workspace_bytes < P.ws)
            return ENGRAM_ENOSPC;
        P.a.x = x;
        P.a.dout = dout;
        P.a.dx = dx;
        P.a.partial = static_cast<float *>(workspace);
        P.a.cu = cu_seqlens;
        P.a.nseq = cu_seqlens != nullptr ? nseq : 1;
        P.a.norm_w = norm_weight;
        P.a.conv_w = conv_weight;
        P.a.bias = conv_bias;
        switch (dtype) {
        case ENGRAM_F32:
            ENGRAM_TRY(launch_conv_bwd_x<float>(P, grad_dtype, s));
            break;
        case ENGRAM_BF16:
            ENGRAM_TRY(launch_conv_bwd_x<__nv_bfloat16>(P, grad_dtype, s));
            break;
        default:
            ENGRAM_TRY(launch_conv_bwd_x<__half>(P, grad_dtype, s));
            break;
        }
    }
    // weight gradients: sum of the blocks' partials (zeros when T = 0)
    int sms = 0;
    ENGRAM_TRY(device_sms(&sms));
    const int64_t work = (int64_t)ple::kBwdQuantities * C;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(ceil_div(work, 256), sms * 4));
    ple::conv_bwd_reduce_kernel<<<blocks, 256, 0, s>>>(
        static_cast<const float *>(workspace), T > 0 ? P.npart : 0, C, K, dconv_weight,
        dconv_bias, dnorm_weight);
    return after_launch();
}

int engram_ple_short_conv_backward(const engram_conv_params_t *params, const void *x,
                                   int32_t dtype, const int32_t *cu_seqlens, int32_t nseq,
                                   int64_t T, const void *norm_weight, const void *conv_weight,
                                   const void *conv_bias, const void *dout, int32_t grad_dtype,
                                   void *dx, float *dnorm_weight, float *dconv_weight,
                                   float *dconv_bias, void *workspace, size_t workspace_bytes,
                                   engram_stream_t stream)
{
    return engram_ple_short_conv_backward_saved(params, x, dtype, cu_seqlens, nseq, T,
                                                norm_weight, conv_weight, conv_bias, nullptr,
                                                dout, grad_dtype, dx, dnorm_weight, dconv_weight,
                                                dconv_bias, workspace, workspace_bytes, stream);
}

} // extern "C"

// ------------------------------------------------------ optimizer step

extern "C" {

int engram_sparse_adam(const engram_adam_params_t *params, void *table, int32_t dtype,
                       int64_t table_rows, int32_t dim, float *exp_avg, float *exp_avg_sq,
                       const int32_t *uniq_rows, const float *row_grads,
                       const int32_t *num_unique, int64_t max_rows, engram_stream_t stream)
{
    if (params == nullptr)
        return ENGRAM_EINVAL;
    const engram_adam_params_t &p = *params;
    const int eb = elem_bytes(dtype);
    if (eb == 0 || dim < 4 || dim % 4 != 0 || table_rows < 1 || table_rows > INT32_MAX ||
        max_rows < 0 || max_rows > INT32_MAX || p.reserved != 0 || p.step < 1)
        return ENGRAM_EINVAL;
    if (!std::isfinite(p.lr) || p.lr < 0.f || !(p.beta1 >= 0.f && p.beta1 < 1.f) ||
        !(p.beta2 >= 0.f && p.beta2 < 1.f) || !std::isfinite(p.eps) || p.eps < 0.f ||
        !std::isfinite(p.weight_decay) || p.weight_decay < 0.f)
        return ENGRAM_EINVAL;
    if (max_rows == 0)
        return ENGRAM_OK;
    if (table == nullptr || exp_avg == nullptr || exp_avg_sq == nullptr ||
        uniq_rows == nullptr || row_grads == nullptr || num_unique == nullptr)
        return ENGRAM_EINVAL;
    if (((uintptr_t)table & (dtype == ENGRAM_F32 ? 15u : 7u)) != 0 || !aligned16(exp_avg) ||
        !aligned16(exp_avg_sq) || !aligned16(row_grads))
        return ENGRAM_EINVAL;
    optim::AdamArgs a;
    a.table = table;
    a.m = exp_avg;
    a.v = exp_avg_sq;
    a.rows = uniq_rows;
    a.grads = row_grads;
    a.num_unique = num_unique;
    a.table_rows = table_rows;
    a.max_rows = max_rows;
    a.dim = dim;
    a.b1 = p.beta1;
    a.b2 = p.beta2;
    a.one_b1 = (float)(1.0 - (double)p.beta1);
    a.one_b2 = (float)(1.0 - (double)p.beta2);
    const double bc1 = 1.0 - std::pow((double)p.beta1, (double)p.step);
    const double bc2 = 1.0 - std::pow((double)p.beta2, (double)p.step);
    a.step_size = (float)((double)p.lr / bc1);
    a.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
    a.eps = p.eps;
    a.decay = (float)(1.0 - (double)p.lr * (double)p.weight_decay);
    int sms = 0;
    ENGRAM_TRY(device_sms(&sms));
    const int64_t work = max_rows * (dim / 4);
    const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>(ceil_div(work, 256), (int64_t)sms * 8));
    cudaStream_t s = (cudaStream_t)stream;
    const bool d160 = dim == 160;
    switch (dtype) {
    case ENGRAM_F32:
        (d160 ? optim::sparse_adam_kernel<float, 40> : optim::sparse_adam_kernel<float, 0>)
            <<<(unsigned)blocks, 256, 0, s>>>(a);
        break;
    case ENGRAM_BF16:
        (d160 ? optim::sparse_adam_kernel<__nv_bfloat16, 40>
              : optim::sparse_adam_kernel<__nv_bfloat16, 0>)<<<(unsigned)blocks, 256, 0, s>>>(a);
        break;
    default:
        (d160 ? optim::sparse_adam_kernel<__half, 40> : optim::sparse_adam_kernel<__half, 0>)
            <<<(unsigned)blocks, 256, 0, s>>>(a);
        break;
    }
    return after_launch();
}

} // extern "C"

// ------------------------------------------------------ owner routing

extern "C" {

int engram_owner_bucket_workspace_size(int64_t n, int32_t owners, size_t *bytes)
{
    if (bytes == nullptr || n < 0 || n > INT32_MAX || owners < 1 || owners > owner::kMaxOwners)
        return ENGRAM_EINVAL;
    const int64_t ntiles = std::max<int64_t>(1, ceil_div(n, owner::kTile));
    *bytes = (size_t)2 * ntiles * owners * sizeof(uint32_t);
    return ENGRAM_OK;
}

} // extern "C"

namespace {

int owner_bucket(const int32_t *rows, int64_t n, int64_t rows_per_owner, int32_t owners,
                 int64_t cap, int32_t *send_rows, int32_t *src_pos, int32_t *dst_pos,
                 int32_t *counts, void *workspace, size_t workspace_bytes, engram_stream_t stream)
{
    size_t need = 0;
    ENGRAM_TRY(engram_owner_bucket_workspace_size(n, owners, &need));
    if (rows_per_owner < 1 || counts == nullptr || cap < 0 || cap > INT32_MAX ||
        cap * owners > INT32_MAX)
        return ENGRAM_EINVAL;
    const int64_t slots = cap > 0 ? cap * owners : n; // grouped positions
    if ((n > 0 && (rows == nullptr || dst_pos == nullptr || workspace == nullptr)) ||
        (slots > 0 && (send_rows == nullptr || src_pos == nullptr)))
        return ENGRAM_EINVAL;
    const size_t nb = (size_t)n * sizeof(int32_t), sb = (size_t)slots * sizeof(int32_t);
    if (overlaps(rows, nb, send_rows, sb) || overlaps(rows, nb, src_pos, sb) ||
        overlaps(rows, nb, dst_pos, nb) || overlaps(send_rows, sb, src_pos, sb) ||
        overlaps(send_rows, sb, dst_pos, nb) || overlaps(src_pos, sb, dst_pos, nb))
        return ENGRAM_EINVAL;
    if (workspace_bytes < need)
        return ENGRAM_ENOSPC;
    owner::OwnerArgs a;
    a.rows = rows;
    a.n = n;
    a.rows_per_owner = rows_per_owner;
    a.owners = owners;
    a.ntiles = (int32_t)std::max<int64_t>(1, ceil_div(n, owner::kTile));
    a.tile_cnt = static_cast<uint32_t *>(workspace);
    a.tile_off = a.tile_cnt + (size_t)a.ntiles * owners;
    a.counts = counts;
    a.send_rows = send_rows;
    a.src_pos = src_pos;
    a.dst_pos = dst_pos;
    a.cap = cap;
    cudaStream_t s = (cudaStream_t)stream;
    if (n > 0) {
        owner::owner_count<<<a.ntiles, owner::kThreads, 0, s>>>(a);
        ENGRAM_TRY(after_launch());
    }
    const int32_t ntiles = a.ntiles;
    if (n == 0)
        a.ntiles = 0;  // counts only: all zero
    owner::owner_scan<<<1, owner::kThreads, 0, s>>>(a);
    ENGRAM_TRY(after_launch());
    a.ntiles = ntiles;
    if (n > 0 || slots > 0) {
        owner::owner_scatter<<<a.ntiles, owner::kThreads, 0, s>>>(a);
        ENGRAM_TRY(after_launch());
    }
    return ENGRAM_OK;
}

} // namespace

extern "C" {

int engram_owner_bucket(const int32_t *rows, int64_t n, int64_t rows_per_owner, int32_t owners,
                        int32_t *send_rows, int32_t *src_pos, int32_t *dst_pos, int32_t *counts,
                        void *workspace, size_t workspace_bytes, engram_stream_t stream)
{
    return owner_bucket(rows, n, rows_per_owner, owners, 0, send_rows, src_pos, dst_pos, counts,
                        workspace, workspace_bytes, stream);
}

int engram_owner_bucket_padded(const int32_t *rows, int64_t n, int64_t rows_per_owner,
                               int32_t owners, int64_t capacity, int32_t *send_rows,
                               int32_t *src_pos, int32_t *dst_pos, int32_t *counts,
                               void *workspace, size_t workspace_bytes, engram_stream_t stream)
{
    if (capacity < 1)
        return ENGRAM_EINVAL;
    return owner_bucket(rows, n, rows_per_owner, owners, capacity, send_rows, src_pos, dst_pos,
                        counts, workspace, workspace_bytes, stream);
}

} // extern "C"
