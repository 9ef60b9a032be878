// norm.cuh -- the branch-local Gemma RMS norm alone (layers page,
// Qwen3_8_FlashNextGroupedRMSNorm; the PLE layer's norm_key / norm_query):
//   out[r, c] = x[r, c] * rsqrt(mean over c's group of x[r, .]^2 + eps) * (1 + w[c])
//
// One block per (group, row range); the (1 + w) scales of the block's group
// sit in shared memory as fp32. Each warp normalises whole group slices: its
// lanes load a slice with 16-byte loads (G * elem / 512 per lane, two slices
// in flight), sum the squares, reduce with shuffles, and write the scaled
// values back with streaming stores. No barrier after the scales are staged,
// no shared-memory traffic for the data: the kernel streams x once and out
// once.
#pragma once

#include "ple_conv.cuh"

namespace engram {
namespace norm {

constexpr int kThreads = 256;
constexpr int kMaxVec = 16;  // 16-byte vectors per lane and slice: G * elem <= 8 KB

struct NormArgs {
    const void *x;
    void *out;
    const void *w;       // [C] of wdtype, or null
    int32_t wdtype;
    int64_t rows;
    int32_t C, G;
    int32_t bpg;         // blocks per group
    float eps, inv_G;
};

template <typename XT, typename OT, int NVEC>
__global__ void __launch_bounds__(kThreads) norm_kernel(const NormArgs a)
{
    constexpr int EV = 16 / (int)sizeof(XT);
    constexpr int OB = EV * (int)sizeof(OT);
    extern __shared__ __align__(16) float scale_s[];  // [G]
    const int m = blockIdx.x / a.bpg, j = blockIdx.x - m * a.bpg;
    for (int c = threadIdx.x; c < a.G; c += blockDim.x)
        scale_s[c] = 1.f + (a.w ? ple::load_weight(a.w, a.wdtype, (int64_t)m * a.G + c) : 0.f);
    __syncthreads();
    const int64_t r0 = a.rows * j / a.bpg, r1 = a.rows * (j + 1) / a.bpg;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int nvec = a.G / EV;  // 16-byte vectors per slice
    const char *xb = static_cast<const char *>(a.x) + (int64_t)m * a.G * sizeof(XT);
    char *ob = static_cast<char *>(a.out) + (int64_t)m * a.G * sizeof(OT);
    const int64_t xrow = (int64_t)a.C * sizeof(XT), orow = (int64_t)a.C * sizeof(OT);
    for (int64_t r = r0 + 2 * wid; r < r1; r += 2 * nw) {
        uint32_t w[2][NVEC][4];
        float ss[2] = {0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int u = 0; u < NVEC; ++u) {
                const int v = u * 32 + lane;
                if (r + h < r1 && v < nvec)
                    ple::load_global<16>(xb + (r + h) * xrow + (size_t)v * 16, w[h][u]);
                else
                    w[h][u][0] = w[h][u][1] = w[h][u][2] = w[h][u][3] = 0u;
            }
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int u = 0; u < NVEC; ++u) {
                float f[EV];
                ple::Elem<XT>::template unpack<EV>(w[h][u], f);
#pragma unroll
                for (int e = 0; e < EV; ++e)
                    ss[h] = fmaf(f[e], f[e], ss[h]);
            }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss[0] += __shfl_xor_sync(kFull, ss[0], o);
            ss[1] += __shfl_xor_sync(kFull, ss[1], o);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            if (r + h >= r1)
                break;
            const float inv = rsqrtf(fmaf(ss[h], a.inv_G, a.eps));
#pragma unroll
            for (int u = 0; u < NVEC; ++u) {
                const int v = u * 32 + lane;
                if (v >= nvec)
                    break;
                float f[EV];
                ple::Elem<XT>::template unpack<EV>(w[h][u], f);
                const float *sc = scale_s + v * EV;
#pragma unroll
                for (int e = 0; e < EV; ++e)
                    f[e] = f[e] * inv * sc[e];
                uint32_t o[OB / 4];
                ple::Elem<OT>::template pack<EV>(f, o);
                ple::store_words<OB>(ob + (r + h) * orow + (size_t)v * OB, o);
            }
        }
    }
}

} // namespace norm
} // namespace engram
