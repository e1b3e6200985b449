// LayerNorm over channels for sm_100a: y = g * (x - mean) / sqrt(var + eps) + b
// per token row, with the biased variance, as applied after the output
// projection of the spatial-mix module ("Vision-RWKV Backbone", Overall
// Architecture).  One warp per row: the row (a few KB) stays in L1 across the
// three passes (mean, centred variance, normalise), so the variance has no
// E[x^2] - E[x]^2 cancellation; HBM sees one read and one write per element.
#pragma once

#include "common.cuh"
#include "qshift.cuh"

namespace vrwkv {

struct LayerNormParams {
    const char* x;
    char* y;
    const float* g;
    const float* b;
    long long rows;
    int C;
    float eps;
    int vec;  // 16-byte vectors (C * sizeof(IO) % 16 == 0, aligned pointers)
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
    return v;
}

// Rows of at most 32 * VPL 16-byte vectors: the warp holds its row in
// registers, so each element is read once; mean and centred variance come
// from the registers.  gamma and beta must be 16-byte aligned.
template <typename IO, int VPL>
__global__ void __launch_bounds__(256) layer_norm_reg_kernel(const LayerNormParams p) {
    using V = Vec16<IO>;
    constexpr int N = V::N;
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= p.rows) return;
    const char* xr = p.x + (size_t)row * p.C * sizeof(IO);
    char* yr = p.y + (size_t)row * p.C * sizeof(IO);
    const int nv = p.C / N;
    float f[VPL][N];
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int v = lane + 32 * k;
        uint4 raw = make_uint4(0u, 0u, 0u, 0u);
        if (v < nv) raw = *reinterpret_cast<const uint4*>(xr + (size_t)v * 16);
        V::unpack(raw, f[k]);
#pragma unroll
        for (int e = 0; e < N; ++e) s += f[k][e];
    }
    const float invC = 1.0f / (float)p.C;
    const float mean = warp_sum(s) * invC;
    float q = 0.f;
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        if (lane + 32 * k < nv) {
#pragma unroll
            for (int e = 0; e < N; ++e) q = fmaf(f[k][e] - mean, f[k][e] - mean, q);
        }
    }
    const float rstd = rsqrtf(warp_sum(q) * invC + p.eps);
#pragma unroll
    for (int k = 0; k < VPL; ++k) {
        const int v = lane + 32 * k;
        if (v < nv) {
            // gamma and beta of the vector's N channels as float4 loads
            const float4* g4 = reinterpret_cast<const float4*>(p.g + v * N);
            const float4* b4 = reinterpret_cast<const float4*>(p.b + v * N);
            float gg[N], bb[N], o[N];
#pragma unroll
            for (int e = 0; e < N / 4; ++e) {
                const float4 a = __ldg(g4 + e), c = __ldg(b4 + e);
                gg[4 * e] = a.x; gg[4 * e + 1] = a.y; gg[4 * e + 2] = a.z; gg[4 * e + 3] = a.w;
                bb[4 * e] = c.x; bb[4 * e + 1] = c.y; bb[4 * e + 2] = c.z; bb[4 * e + 3] = c.w;
            }
#pragma unroll
            for (int e = 0; e < N; ++e) o[e] = fmaf(gg[e], (f[k][e] - mean) * rstd, bb[e]);
            *reinterpret_cast<uint4*>(yr + (size_t)v * 16) = V::pack(o);
        }
    }
}

template <typename IO>
__global__ void __launch_bounds__(256) layer_norm_kernel(const LayerNormParams p) {
    using V = Vec16<IO>;
    constexpr int N = V::N;
    const int lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= p.rows) return;
    const char* xr = p.x + (size_t)row * p.C * sizeof(IO);
    char* yr = p.y + (size_t)row * p.C * sizeof(IO);
    const float invC = 1.0f / (float)p.C;
    float s = 0.f;
    if (p.vec) {
        const int nv = p.C / N;
        for (int v = lane; v < nv; v += 32) {
            float f[N];
            V::unpack(*reinterpret_cast<const uint4*>(xr + (size_t)v * 16), f);
#pragma unroll
            for (int e = 0; e < N; ++e) s += f[e];
        }
        const float mean = warp_sum(s) * invC;
        float q = 0.f;
        for (int v = lane; v < nv; v += 32) {
            float f[N];
            V::unpack(*reinterpret_cast<const uint4*>(xr + (size_t)v * 16), f);
#pragma unroll
            for (int e = 0; e < N; ++e) q = fmaf(f[e] - mean, f[e] - mean, q);
        }
        const float rstd = rsqrtf(warp_sum(q) * invC + p.eps);
        for (int v = lane; v < nv; v += 32) {
            float f[N], o[N];
            V::unpack(*reinterpret_cast<const uint4*>(xr + (size_t)v * 16), f);
#pragma unroll
            for (int e = 0; e < N; ++e) {
                const int c = v * N + e;
                o[e] = fmaf(__ldg(p.g + c), (f[e] - mean) * rstd, __ldg(p.b + c));
            }
            *reinterpret_cast<uint4*>(yr + (size_t)v * 16) = V::pack(o);
        }
    } else {
        for (int c = lane; c < p.C; c += 32) s += Io<IO>::ld1(xr + (size_t)c * sizeof(IO));
        const float mean = warp_sum(s) * invC;
        float q = 0.f;
        for (int c = lane; c < p.C; c += 32) {
            const float d = Io<IO>::ld1(xr + (size_t)c * sizeof(IO)) - mean;
            q = fmaf(d, d, q);
        }
        const float rstd = rsqrtf(warp_sum(q) * invC + p.eps);
        for (int c = lane; c < p.C; c += 32) {
            const float d = Io<IO>::ld1(xr + (size_t)c * sizeof(IO)) - mean;
            Io<IO>::st1(yr + (size_t)c * sizeof(IO), fmaf(__ldg(p.g + c), d * rstd, __ldg(p.b + c)));
        }
    }
}

}  // namespace vrwkv
