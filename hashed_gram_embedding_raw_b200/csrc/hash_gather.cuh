// hash_gather.cuh -- N-gram hash, row gather, and the fused hash+gather kernel.
//
// Qwen3.8-Flash-Next engram API page, class Qwen3_8_FlashNextNGramEmbedding:
// _shift_right_after_eos (earlier tokens without crossing an EOS),
// _hash_input_ids (signed int64 products of the earlier tokens with the layer
// multipliers, positive remainder by each head's prime, plus the head's global
// offset; bigram heads first) and _lookup_ngram_ids / forward (rows of the
// packed table concatenated over heads).
//
// Work split: the T tokens are cut into one contiguous range per warp
// (balanced to one token), and each warp walks its range 32 tokens at a time,
// one token per lane. The previous one to three tokens come from warp
// shuffles (lanes 0..2 read their halo from global memory), the EOS/sequence
// reset is evaluated per lane from those same registers plus the warp's
// cursor into cu_seqlens, and the H row indices of the 32 tokens go to a
// small per-warp shared-memory tile. The gather then streams rows as 16-byte
// vectors: for each token, lane l moves vectors l, l+32, ... of the token's
// H*V vector output (V = 16-byte vectors per row), so every store
// instruction writes 512 contiguous bytes and the reads cover whole 32-byte
// sectors of each 64-byte-aligned row.
#pragma once

#include "common.cuh"

namespace engram {

struct HashArgs {
    int32_t N, K, H, eos;
    int64_t fill;
    int64_t mult[ENGRAM_MAX_NGRAM];
    uint64_t p[ENGRAM_MAX_HEADS];
    uint64_t magic[ENGRAM_MAX_HEADS];
    int32_t off[ENGRAM_MAX_HEADS];
};

constexpr int kHashThreads = 256;

// A slice of the stream (_forward_global_slice): positions [start, start+len)
// of every row of `row` tokens. Logical token L of the slice is stream
// position (L / len) * row + start + L % len; the identity map has row = len
// = 1 << 62, start = 0.
struct SliceMap {
    int64_t row, start, len;
};

__device__ __forceinline__ int64_t slice_token(const SliceMap &m, int64_t L)
{
    return (L / m.len) * m.row + m.start + L % m.len;
}

// Hashes logical tokens l0 .. l0+31 below l_end (lane i owns l0 + i) and
// writes their H row indices to s_idx[i * HP + h]. Without MAPPED the logical
// token is the stream position and the earlier tokens come from neighbouring
// lanes; with MAPPED the position comes from the slice map and earlier tokens
// are read from global memory (the whole stream is there, so context from
// before the slice is kept). `s` is the warp's cursor into cu_seqlens: on
// entry cu[s] <= the chunk's first position; on exit s is the largest index
// below nseq whose bound is <= the chunk's last position.
template <int NT, int KT, bool MAPPED = false>
__device__ __forceinline__ void hash_chunk(const HashArgs &a, const int32_t *__restrict__ ids,
                                           const int32_t *__restrict__ cu, int32_t nseq,
                                           int64_t T, int64_t l0, int64_t l_end, int32_t &s,
                                           int32_t *s_idx, int HP, int lane,
                                           const SliceMap &m = SliceMap{0, 0, 1})
{
    const int N = NT ? NT : a.N;
    const int K = KT ? KT : a.K;
    const int64_t L = l0 + lane;
    const int64_t t = MAPPED ? slice_token(m, min(L, l_end - 1)) : L;
    const int32_t x0 = L < l_end ? __ldg(ids + t) : 0;

    // Start of the lane's sequence: sequence bounds inside this chunk are
    // visited in order, each lane keeping the last one at or before its token.
    int64_t S = 0;
    if (cu != nullptr) {
        S = __ldg(cu + s);
        const int64_t llast = min(l0 + 31, l_end - 1);
        const int64_t last = MAPPED ? slice_token(m, llast) : llast;
        while (s + 1 < nseq) {
            const int64_t b = __ldg(cu + s + 1);
            if (b > last)
                break;
            ++s;
            if (t >= b)
                S = b;
        }
    }

    // x[k]: the token k places back, or fill when a reset lies in between
    // (sequence start, or an EOS at any of positions t-k .. t-1).
    int64_t x[ENGRAM_MAX_NGRAM];
    x[0] = x0;
    bool ok = true;
#pragma unroll
    for (int k = 1; k < ENGRAM_MAX_NGRAM; ++k) {
        if (k < N) {
            int32_t prev;
            if constexpr (MAPPED) {
                prev = t - k >= 0 ? __ldg(ids + t - k) : 0;
            } else {
                prev = __shfl_up_sync(kFull, x0, k);
                if (lane < k)
                    prev = (t - k >= 0 && t - k < T) ? __ldg(ids + t - k) : 0;
            }
            ok = ok && (t - k >= S) && (prev != a.eos);
            x[k] = ok ? (int64_t)prev : a.fill;
        }
    }

    // Order-n mix = XOR of the wrapped products of the n most recent tokens.
    int64_t mix = (int64_t)((uint64_t)x[0] * (uint64_t)a.mult[0]);
    int32_t *row = s_idx + lane * HP;
#pragma unroll
    for (int g = 0; g < ENGRAM_MAX_NGRAM - 1; ++g) {
        if (g < N - 1) {
            mix ^= (int64_t)((uint64_t)x[g + 1] * (uint64_t)a.mult[g + 1]);
            if constexpr (KT != 0) {
#pragma unroll
                for (int i = 0; i < KT; ++i) {
                    const int h = g * KT + i;
                    row[h] = a.off[h] + (int32_t)floor_mod(mix, a.p[h], a.magic[h]);
                }
            } else {
                for (int i = 0; i < K; ++i) {
                    const int h = g * K + i;
                    row[h] = a.off[h] + (int32_t)floor_mod(mix, a.p[h], a.magic[h]);
                }
            }
        }
    }
}

// Token range [tb, te) of warp w out of nwarps, balanced to one token.
__device__ __forceinline__ void warp_range(int64_t total, int64_t w, int64_t nwarps,
                                           int64_t &b, int64_t &e)
{
    b = total * w / nwarps;
    e = total * (w + 1) / nwarps;
}

// engram_hash: row indices only, out_idx [T, H] int32.
template <int NT, int KT>
__global__ void __launch_bounds__(kHashThreads)
    hash_kernel(HashArgs a, const int32_t *__restrict__ ids, const int32_t *__restrict__ cu,
                int32_t nseq, int64_t T, int64_t nwarps, int32_t *__restrict__ out_idx)
{
    extern __shared__ int32_t smem[];
    if (cu != nullptr)
        check_cu_seqlens(cu, nseq, T);
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    const int H = ((NT ? NT : a.N) - 1) * (KT ? KT : a.K);
    const int HP = H + 1;
    int32_t *s_idx = smem + wib * 32 * HP;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib;
    if (w >= nwarps)
        return;
    int64_t tb, te;
    warp_range(T, w, nwarps, tb, te);
    int32_t s = cu != nullptr ? find_sequence_warp(cu, nseq, tb) : 0;
    for (int64_t t0 = tb; t0 < te; t0 += 32) {
        hash_chunk<NT, KT>(a, ids, cu, nseq, T, t0, te, s, s_idx, HP, lane);
        __syncwarp();
        const int ntok = (int)min64(32, te - t0);
        for (int e = lane; e < ntok * H; e += 32)
            out_idx[t0 * H + e] = s_idx[(e / H) * HP + e % H];
        __syncwarp();
    }
}

// engram_hash_gather: hash a chunk, then stream its rows.
// VT = 16-byte vectors per row (20 for bf16 x 160, 40 for fp32 x 160); 0 = runtime.
// MAPPED: hash and gather only the slice described by m (nlog logical tokens
// of the T-token stream); outputs are indexed by logical token.
template <int NT, int KT, int VT, bool MAPPED = false>
__global__ void __launch_bounds__(kHashThreads)
    hash_gather_kernel(HashArgs a, const int32_t *__restrict__ ids,
                       const int32_t *__restrict__ cu, int32_t nseq, int64_t T, int64_t nwarps,
                       const uint4 *__restrict__ table, int v_rt,
                       int32_t *__restrict__ out_idx, uint4 *__restrict__ out,
                       SliceMap m = SliceMap{0, 0, 1}, int64_t nlog = 0)
{
    extern __shared__ int32_t smem[];
    if (cu != nullptr)
        check_cu_seqlens(cu, nseq, T);
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    constexpr int HT = (NT && KT) ? (NT - 1) * KT : 0;
    const int H = HT ? HT : (a.N - 1) * a.K;
    const int HP = H + 1;
    const int V = VT ? VT : v_rt;
    int32_t *s_idx = smem + wib * 32 * HP;
    const int64_t w = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib;
    if (w >= nwarps)
        return;
    int64_t tb, te;
    warp_range(MAPPED ? nlog : T, w, nwarps, tb, te);
    if (tb >= te)
        return;
    int32_t s = cu != nullptr ? find_sequence_warp(cu, nseq, MAPPED ? slice_token(m, tb) : tb)
                              : 0;

    for (int64_t t0 = tb; t0 < te; t0 += 32) {
        hash_chunk<NT, KT, MAPPED>(a, ids, cu, nseq, T, t0, te, s, s_idx, HP, lane, m);
        __syncwarp();
        const int ntok = (int)min64(32, te - t0);
        if (out_idx != nullptr)
            for (int e = lane; e < ntok * H; e += 32)
                out_idx[t0 * H + e] = s_idx[(e / H) * HP + e % H];

        if constexpr (HT != 0 && VT != 0 && (HT * VT) % 32 == 0) {
            // Fixed shape: every lane moves PER vectors per token, UNROLL
            // tokens' loads in flight before their stores.
            constexpr int PER = HT * VT / 32;
            constexpr int UNROLL = PER <= 10 ? 2 : 1;
            for (int j = 0; j < ntok; j += UNROLL) {
                uint4 v[UNROLL][PER];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int tok = j + u;
                    if (tok < ntok) {
#pragma unroll
                        for (int q = 0; q < PER; ++q) {
                            const int k = lane + 32 * q;
                            const int h = k / VT, c = k - h * VT;
                            const int32_t r = s_idx[tok * HP + h];
                            v[u][q] = ld_stream(table + (size_t)r * VT + c);
                        }
                    }
                }
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int tok = j + u;
                    if (tok < ntok) {
                        uint4 *dst = out + (size_t)(t0 + tok) * (HT * VT);
#pragma unroll
                        for (int q = 0; q < PER; ++q)
                            st_stream(dst + lane + 32 * q, v[u][q]);
                    }
                }
            }
        } else {
            const int per_tok = H * V;
            for (int tok = 0; tok < ntok; ++tok) {
                uint4 *dst = out + (size_t)(t0 + tok) * per_tok;
                for (int k = lane; k < per_tok; k += 32) {
                    const int h = k / V, c = k - h * V;
                    const int32_t r = s_idx[tok * HP + h];
                    st_stream(dst + k, ld_stream(table + (size_t)r * V + c));
                }
            }
        }
        __syncwarp();
    }
}

// engram_gather: out[i] = table[idx[i]] for n lookups of V 16-byte vectors
// (a zero row where idx[i] < 0).
// A warp moves 32 rows at a time: lane l handles vectors l, l+32, ... of the
// 32 x V chunk, taking each vector's row index from the owning lane by
// shuffle, so stores stay fully coalesced for any V.
template <int VT>
__global__ void __launch_bounds__(kHashThreads, 2)
    gather_kernel(const uint4 *__restrict__ table, int64_t rows, int v_rt,
                  const int32_t *__restrict__ idx, int64_t n, int64_t nwarps,
                  uint4 *__restrict__ out)
{
    const int lane = threadIdx.x & 31;
    const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (w >= nwarps)
        return;
    const int V = VT ? VT : v_rt;
    int64_t ib, ie;
    warp_range(n, w, nwarps, ib, ie);
    for (int64_t i0 = ib; i0 < ie; i0 += 32) {
        const int nrow = (int)min64(32, ie - i0);
        // a negative index marks an absent lookup (padding): a zero row; an
        // index past the table is an error, also answered with a zero row
        int32_t my = lane < nrow ? __ldg(idx + i0 + lane) : 0;
        if (lane < nrow && (int64_t)my >= rows)
            raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
        if (my < 0 || (int64_t)my >= rows)
            my = -1;
        uint4 *dst = out + (size_t)i0 * V;
        if constexpr (VT != 0) {
            constexpr int BATCH = VT < 20 ? VT : 20;   // vectors in flight per lane
#pragma unroll
            for (int q0 = 0; q0 < VT; q0 += BATCH) {
                uint4 v[BATCH];
#pragma unroll
                for (int q = 0; q < BATCH; ++q) {
                    const int k = lane + 32 * (q0 + q);
                    const int r = k / VT, c = k - r * VT;
                    const int32_t row = __shfl_sync(kFull, my, r);
                    v[q] = make_uint4(0, 0, 0, 0);
                    if (r < nrow && row >= 0)
                        v[q] = ld_stream(table + (size_t)row * VT + c);
                }
#pragma unroll
                for (int q = 0; q < BATCH; ++q) {
                    const int k = lane + 32 * (q0 + q);
                    if (k / VT < nrow)
                        st_stream(dst + k, v[q]);
                }
            }
        } else {
            for (int k = lane; k < 32 * V; k += 32) {
                const int r = k / V, c = k - r * V;
                const int32_t row = __shfl_sync(kFull, my, r);
                if (r < nrow)
                    st_stream(dst + k, row >= 0 ? ld_stream(table + (size_t)row * V + c)
                                                : make_uint4(0, 0, 0, 0));
            }
        }
    }
}

} // namespace engram
