// optim.cuh -- the optimizer step on the rows a backward produced: AdamW
// with per-row first and second moments, updated only on those rows (the
// owner "stores and updates each row's gradient", model card; the table's
// optimizer tensors live in the checkpoint, model card §Current Scope).
//
// For u < U = min(*num_unique, max_rows), r = rows[u], g = grads[u, :]:
//   p[r] *= 1 - lr * wd
//   m[r]  = b1 * m[r] + (1 - b1) * g
//   v[r]  = b2 * v[r] + (1 - b2) * g^2
//   p[r] -= lr / (1 - b1^step) * m[r] / (sqrt(v[r]) / sqrt(1 - b2^step) + eps)
// The kernel reads U from device memory (the backward's num_unique), so no
// host round trip separates the backward from the step. One thread updates
// four columns of one row (16 bytes of g, m, v; 8 or 16 bytes of p), threads
// are consecutive along a row, and the grid strides over rows x column
// groups: every access is coalesced within a row, and the rows themselves
// are random. HBM-bound: 3,844 bytes per 160-wide bf16 row.
#pragma once

#include "common.cuh"

namespace engram {
namespace optim {

struct AdamArgs {
    void *table;
    float *m, *v;
    const int32_t *rows;
    const float *grads;
    const int32_t *num_unique;
    int64_t table_rows, max_rows;
    int32_t dim;
    float b1, b2, one_b1, one_b2;  // betas and 1 - betas
    float step_size;               // lr / (1 - b1^step)
    float inv_sqrt_bc2;            // 1 / sqrt(1 - b2^step)
    float eps, decay;              // eps, 1 - lr * wd
};

__device__ __forceinline__ float4 ld_f4(const float *p)
{
    return *reinterpret_cast<const float4 *>(p);
}

__device__ __forceinline__ void st_f4(float *p, float4 v)
{
    *reinterpret_cast<float4 *>(p) = v;
}

template <typename PT>
struct Param4;

template <>
struct Param4<float> {
    __device__ static float4 load(const void *t, int64_t i)
    {
        return *reinterpret_cast<const float4 *>(static_cast<const float *>(t) + i);
    }
    __device__ static void store(void *t, int64_t i, float4 v)
    {
        *reinterpret_cast<float4 *>(static_cast<float *>(t) + i) = v;
    }
};

template <>
struct Param4<__nv_bfloat16> {
    __device__ static float4 load(const void *t, int64_t i)
    {
        const uint2 w = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(t) + i);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
    }
    __device__ static void store(void *t, int64_t i, float4 v)
    {
        uint2 w;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.x) : "f"(v.y), "f"(v.x));
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w.y) : "f"(v.w), "f"(v.z));
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(t) + i) = w;
    }
};

template <>
struct Param4<__half> {
    __device__ static float4 load(const void *t, int64_t i)
    {
        const uint2 w = *reinterpret_cast<const uint2 *>(static_cast<const uint16_t *>(t) + i);
        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&w.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&w.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    __device__ static void store(void *t, int64_t i, float4 v)
    {
        uint2 w;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w.x) : "f"(v.y), "f"(v.x));
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(w.y) : "f"(v.w), "f"(v.z));
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(t) + i) = w;
    }
};

__device__ __forceinline__ float adam1(float &p, float &m, float &v, float g, const AdamArgs &a)
{
    p *= a.decay;
    m = fmaf(a.b1, m, a.one_b1 * g);
    v = fmaf(a.b2, v, a.one_b2 * (g * g));
    const float denom = fmaf(sqrtf(v), a.inv_sqrt_bc2, a.eps);
    p -= a.step_size * (m / denom);
    return p;
}

// VT: column groups of four per row (40 for dim 160; 0 = runtime dim / 4).
template <typename PT, int VT>
__global__ void __launch_bounds__(256) sparse_adam_kernel(const AdamArgs a)
{
    const int V = VT ? VT : a.dim / 4;
    const int64_t U = min64(a.max_rows, (int64_t)max(0, __ldg(a.num_unique)));
    const int64_t total = U * V;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    bool bad = false;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += stride) {
        const int64_t u = e / V;
        const int c = (int)(e - u * V) * 4;
        const int32_t r = __ldg(a.rows + u);
        if (r < 0 || r >= a.table_rows) {
            bad = true;
            continue;
        }
        const int64_t pi = (int64_t)r * a.dim + c;
        const float4 g = __ldg(reinterpret_cast<const float4 *>(a.grads + u * a.dim + c));
        float4 m = ld_f4(a.m + pi), v = ld_f4(a.v + pi);
        float4 p = Param4<PT>::load(a.table, pi);
        adam1(p.x, m.x, v.x, g.x, a);
        adam1(p.y, m.y, v.y, g.y, a);
        adam1(p.z, m.z, v.z, g.z, a);
        adam1(p.w, m.w, v.w, g.w, a);
        st_f4(a.m + pi, m);
        st_f4(a.v + pi, v);
        Param4<PT>::store(a.table, pi, p);
    }
    if (bad)
        raise_device_error(ENGRAM_DEVERR_ROW_RANGE);
}

} // namespace optim
} // namespace engram
