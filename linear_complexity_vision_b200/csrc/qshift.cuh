// Q-Shift kernel ("Vision-RWKV Backbone", Quad-Directional Token Shift,
// eq. 9, with the channel-group layout of the q_shift listing on
// "LinXin's Blog").  One thread handles one 16-byte vector of channels of one
// token: one coalesced load of x, one load of the shifted neighbour (an L1/L2
// hit: the same rows are read as x by neighbouring threads), one store.
#pragma once

#include "common.cuh"

namespace vrwkv {

// 16-byte vectors of the storage type, unpacked to float32.
template <typename IO>
struct Vec16;

template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ __forceinline__ static void unpack(uint4 r, float (&f)[N]) {
        f[0] = __uint_as_float(r.x); f[1] = __uint_as_float(r.y);
        f[2] = __uint_as_float(r.z); f[3] = __uint_as_float(r.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[N]) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                          __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};

template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ __forceinline__ static void unpack(uint4 r, float (&f)[N]) {
        const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint32_t pack2(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[N]) {
        return make_uint4(pack2(f[0], f[1]), pack2(f[2], f[3]), pack2(f[4], f[5]),
                          pack2(f[6], f[7]));
    }
};

// mu*x + (1-mu)*x_shift with each operation rounded on its own.
__device__ __forceinline__ float qs_mix(float mu, float x, float xd) {
    float t1 = __fmul_rn(mu, x);
    float om = __fsub_rn(1.0f, mu);
    float t2 = __fmul_rn(om, xd);
    return __fadd_rn(t1, t2);
}

struct QshiftParams {
    const char* x;
    char* out;
    const float* mu;  // nullable
    long long BT;     // B*T
    int T, C, H, W, s;
    QsBounds g;       // channel-group bounds
    int ng;           // shifted groups: 4 (Q-Shift) or 2 (bidirectional shift)
};

// Vector path: C*sizeof(IO) is a multiple of 16 and both pointers are
// 16-byte aligned.
template <typename IO>
__global__ void __launch_bounds__(256) qshift_vec_kernel(const QshiftParams p) {
    using V = Vec16<IO>;
    constexpr int N = V::N;
    const int UR = p.C / N;  // vectors per token row
    const long long units = p.BT * UR;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < units;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long bt = idx / UR;
        const int c = (int)(idx - bt * UR) * N;
        const int t = (int)(bt % p.T);
        const int h = t / p.W, w = t - (t / p.W) * p.W;
        const size_t row = (size_t)bt * p.C;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p.x + (row + c) * sizeof(IO)));
        float xv[N], xd[N];
        V::unpack(raw, xv);
        const ShiftRule r0 = shift_rule(c, p.g, p.ng, p.H, p.W, p.s);
        const ShiftRule r1 = shift_rule(c + N - 1, p.g, p.ng, p.H, p.W, p.s);
        if (r0.off == r1.off && r0.use_w == r1.use_w && r0.lo == r1.lo && r0.hi == r1.hi) {
            if (shift_ok(r0, h, w)) {
                const uint4 rd = __ldg(reinterpret_cast<const uint4*>(
                    p.x + (row + (long long)r0.off * p.C + c) * sizeof(IO)));
                V::unpack(rd, xd);
            } else {
#pragma unroll
                for (int e = 0; e < N; ++e) xd[e] = 0.0f;
            }
        } else {  // the vector straddles a channel-group boundary
#pragma unroll
            for (int e = 0; e < N; ++e) {
                const ShiftRule re = shift_rule(c + e, p.g, p.ng, p.H, p.W, p.s);
                xd[e] = shift_ok(re, h, w)
                            ? Io<IO>::ld1(p.x + (row + (long long)re.off * p.C + c + e) * sizeof(IO))
                            : 0.0f;
            }
        }
        float o[N];
        if (p.mu) {
#pragma unroll
            for (int e = 0; e < N; ++e) o[e] = qs_mix(__ldg(p.mu + c + e), xv[e], xd[e]);
        } else {
#pragma unroll
            for (int e = 0; e < N; ++e) o[e] = xd[e];
        }
        *reinterpret_cast<uint4*>(p.out + (row + c) * sizeof(IO)) = V::pack(o);
    }
}

// Scalar path for any C and any element-aligned pointers.
template <typename IO>
__global__ void __launch_bounds__(256) qshift_scalar_kernel(const QshiftParams p) {
    const long long n = p.BT * p.C;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long bt = idx / p.C;
        const int c = (int)(idx - bt * p.C);
        const int t = (int)(bt % p.T);
        const int h = t / p.W, w = t - (t / p.W) * p.W;
        const ShiftRule r = shift_rule(c, p.g, p.ng, p.H, p.W, p.s);
        const float xd = shift_ok(r, h, w)
                             ? Io<IO>::ld1(p.x + (idx + (long long)r.off * p.C) * sizeof(IO))
                             : 0.0f;
        float o = xd;
        if (p.mu) o = qs_mix(__ldg(p.mu + c), Io<IO>::ld1(p.x + idx * sizeof(IO)), xd);
        Io<IO>::st1(p.out + idx * sizeof(IO), o);
    }
}

}  // namespace vrwkv
