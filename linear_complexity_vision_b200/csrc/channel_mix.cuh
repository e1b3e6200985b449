// Channel-mix elementwise path ("Vision-RWKV Backbone", Overall Architecture,
// eq. 3-4, with identity W_R, W_K, W_V and no W_O):
//   out = sigma(QS_R(x)) (.) SquaredReLU(QS_K(x)),  SquaredReLU(z) = max(z, 0)^2,
// where QS_* is Q-Shift (Quad-Directional Token Shift, eq. 9) with mu_r or
// mu_k.  Both mixes read the same shifted neighbour x_shift, so one load of x
// and one of x_shift feed both.
//
// The work is HBM-bound: per element one read of x and one write of out (the
// neighbour load is an L2 hit, since nearby rows are read as x by CTAs that
// run at the same time).  Shared memory and L1 deliver 128 B/clk/SM, too
// little to fetch mu_r and mu_k for every element, so each thread owns ONE
// fixed 16-byte vector of channels, keeps its mu values in registers and walks
// a contiguous range of token rows, four rows in flight at a time (two
// batches of two, software-pipelined).
#pragma once

#include "common.cuh"
#include "qshift.cuh"

namespace vrwkv {

// Unsigned division by a run-time invariant d >= 1 for dividends n < 2^31,
// as a multiply and a shift (Granlund and Montgomery, "Division by Invariant
// Integers using Multiplication", PLDI 1994, Theorem 4.2 with N = 31):
// with l = ceil(log2 d) and m = ceil(2^(31+l) / d), m*d - 2^(31+l) < d <= 2^l,
// so floor(n/d) = floor(m*n / 2^(31+l)); m < 2^32 for every d < 2^31.
struct FastDiv {
    unsigned int m;
    int shift;  // 31 + l
    unsigned int d;
};

inline FastDiv make_fastdiv(unsigned int d) {
    int l = 0;
    while ((1ull << l) < d) ++l;
    const unsigned long long p = 1ull << (31 + l);
    FastDiv f;
    f.m = (unsigned int)((p + d - 1) / d);
    f.shift = 31 + l;
    f.d = d;
    return f;
}

__device__ __forceinline__ unsigned int fdiv(unsigned int n, const FastDiv& f) {
    return (unsigned int)(((unsigned long long)f.m * n) >> f.shift);
}

struct ChannelMixParams {
    const char* x;
    char* out;
    const float* mu_r;  // nullable: QS_R(x) = x_shift
    const float* mu_k;  // nullable: QS_K(x) = x_shift
    int BT;             // B*T token rows, < 2^31
    int T, C, H, W, s;
    QsBounds g;         // Q-Shift channel-group bounds
    int ng;             // shifted groups: 4 (Q-Shift) or 2 (bidirectional shift)
    int UR;             // 16-byte vectors per token row
    FastDiv divT, divW;
};

constexpr int kCmRows = 2;  // token rows per load batch; two batches in flight

template <typename IO>
struct CmColumn {
    using V = Vec16<IO>;
    static constexpr int N = V::N;
    const ChannelMixParams& p;
    ShiftRule rule;
    float2 mur[N / 2], muk[N / 2];
    const char* xcol;
    char* ocol;
    size_t rowb;
    int r1, ty;

    // Loads x and x_shift of rows base, base+ty, ... (rows >= r1 read nothing).
    __device__ __forceinline__ void load(int base, uint4 (&rx)[kCmRows], uint4 (&rd)[kCmRows]) const {
#pragma unroll
        for (int j = 0; j < kCmRows; ++j) {
            const int r = base + j * ty;
            rx[j] = make_uint4(0u, 0u, 0u, 0u);
            rd[j] = make_uint4(0u, 0u, 0u, 0u);
            if (r < r1) {
                const unsigned int t = (unsigned int)r - fdiv((unsigned int)r, p.divT) * (unsigned int)p.T;
                const int h = (int)fdiv(t, p.divW);
                const int w = (int)t - h * p.W;
                rx[j] = __ldg(reinterpret_cast<const uint4*>(xcol + (size_t)r * rowb));
                if (shift_ok(rule, h, w))
                    rd[j] = __ldg(reinterpret_cast<const uint4*>(xcol + (size_t)(r + rule.off) * rowb));
            }
        }
    }

    __device__ __forceinline__ void compute(int base, const uint4 (&rx)[kCmRows],
                                            const uint4 (&rd)[kCmRows]) const {
#pragma unroll
        for (int j = 0; j < kCmRows; ++j) {
            const int r = base + j * ty;
            if (r >= r1) break;
            float xv[N], xd[N], o[N];
            V::unpack(rx[j], xv);
            V::unpack(rd[j], xd);
#pragma unroll
            for (int e = 0; e < N / 2; ++e) {
                const float2 X = f2(xv[2 * e], xv[2 * e + 1]);
                const float2 D = f2(xd[2 * e], xd[2 * e + 1]);
                const float2 dif = fma2(D, f2(-1.0f), X);
                const float2 rr = fma2(mur[e], dif, D);
                const float2 kk = fma2(muk[e], dif, D);
                // sigma(r) = 1 / (1 + 2^(-r*log2 e)); r -> -inf gives 1/inf = 0
                const float2 den = add2(ex2(mul2(rr, f2(-kLog2e))), f2(1.0f));
                const float2 kp = max2(kk, f2(0.0f));
                const float2 y = mul2(mul2(kp, kp), rcp(den));
                o[2 * e] = y.x;
                o[2 * e + 1] = y.y;
            }
            __stcs(reinterpret_cast<uint4*>(ocol + (size_t)r * rowb), V::pack(o));
        }
    }
};

// Vector path: C*sizeof(IO) is a multiple of 16, x and out are 16-byte aligned
// and no vector straddles a channel-group boundary (g is a multiple of the
// vector width, or g == 0).  blockDim = (tx, ty): threadIdx.x picks the
// vector within a channel chunk of tx vectors (blockIdx.x), threadIdx.y the
// row within a group of ty consecutive rows.  blockIdx.y owns the contiguous
// token-row range [BT*by/Gy, BT*(by+1)/Gy), so every CTA moves the same bytes.
// The loads of the next batch of rows are issued before the current batch is
// computed (two register sets), keeping four row loads per thread in flight.
template <typename IO>
__global__ void __launch_bounds__(256, 3) channel_mix_vec_kernel(const ChannelMixParams p) {
    constexpr int N = Vec16<IO>::N;
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= p.UR) return;
    const int c0 = v * N;

    CmColumn<IO> col{p};
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
        col.mur[e] = p.mu_r ? __ldg(reinterpret_cast<const float2*>(p.mu_r + c0) + e) : f2(0.0f);
        col.muk[e] = p.mu_k ? __ldg(reinterpret_cast<const float2*>(p.mu_k + c0) + e) : f2(0.0f);
    }
    // Without mu the mix, xd + mu*(x - xd), is xd itself.
    col.rule = shift_rule(c0, p.g, p.ng, p.H, p.W, p.s);
    const long long Gy = gridDim.y;
    const int r0 = (int)((long long)p.BT * blockIdx.y / Gy);
    col.r1 = (int)((long long)p.BT * (blockIdx.y + 1) / Gy);
    col.ty = blockDim.y;
    col.rowb = (size_t)p.C * sizeof(IO);
    col.xcol = p.x + (size_t)c0 * sizeof(IO);
    col.ocol = p.out + (size_t)c0 * sizeof(IO);

    const int step = col.ty * kCmRows;
    uint4 ax[kCmRows], ad[kCmRows], bx[kCmRows], bd[kCmRows];
    int base = r0 + threadIdx.y;
    col.load(base, ax, ad);
    for (; base < col.r1; base += 2 * step) {
        col.load(base + step, bx, bd);
        col.compute(base, ax, ad);
        if (base + step >= col.r1) break;
        col.load(base + 2 * step, ax, ad);
        col.compute(base + step, bx, bd);
    }
}

// Q-Shift mixes on the same column walk: NMIX outputs out[m] = mu_m*x +
// (1-mu_m)*x_shift (t1 = mu*x, t2 = (1-mu)*x_shift, t1 + t2, each rounded, as
// qshift_vec_kernel), or x_shift itself when mu[0] is null (NMIX = 1).  One
// load of x and of its neighbour feeds every output.  Requires the vector
// conditions of channel_mix_vec_kernel (no vector straddles a channel group).
template <int NMIX>
struct QsMixParams {
    ChannelMixParams base;  // x, BT, T, C, H, W, s, g, UR, divT, divW
    char* out[NMIX];
    const float* mu[NMIX];
};

template <typename IO, int NMIX>
__global__ void __launch_bounds__(256) qs_mix_vec_kernel(const QsMixParams<NMIX> q) {
    using V = Vec16<IO>;
    constexpr int N = V::N;
    const ChannelMixParams& p = q.base;
    const int v = blockIdx.x * blockDim.x + threadIdx.x;
    if (v >= p.UR) return;
    const int c0 = v * N;
    const bool with_mu = q.mu[0] != nullptr;
    float mu[NMIX][N];
#pragma unroll
    for (int m = 0; m < NMIX; ++m)
#pragma unroll
        for (int e = 0; e < N; ++e) mu[m][e] = with_mu ? __ldg(q.mu[m] + c0 + e) : 0.0f;
    const ShiftRule rule = shift_rule(c0, p.g, p.ng, p.H, p.W, p.s);
    const long long Gy = gridDim.y;
    const int r0 = (int)((long long)p.BT * blockIdx.y / Gy);
    const int r1 = (int)((long long)p.BT * (blockIdx.y + 1) / Gy);
    const int ty = blockDim.y;
    const size_t rowb = (size_t)p.C * sizeof(IO);
    const char* xcol = p.x + (size_t)c0 * sizeof(IO);
    for (int base = r0 + threadIdx.y; base < r1; base += ty * kCmRows) {
        uint4 rx[kCmRows], rd[kCmRows];
#pragma unroll
        for (int j = 0; j < kCmRows; ++j) {
            const int r = base + j * ty;
            rx[j] = make_uint4(0u, 0u, 0u, 0u);
            rd[j] = make_uint4(0u, 0u, 0u, 0u);
            if (r < r1) {
                const unsigned int t = (unsigned int)r - fdiv((unsigned int)r, p.divT) * (unsigned int)p.T;
                const int h = (int)fdiv(t, p.divW);
                const int w = (int)t - h * p.W;
                rx[j] = __ldg(reinterpret_cast<const uint4*>(xcol + (size_t)r * rowb));
                if (shift_ok(rule, h, w))
                    rd[j] = __ldg(reinterpret_cast<const uint4*>(xcol + (size_t)(r + rule.off) * rowb));
            }
        }
#pragma unroll
        for (int j = 0; j < kCmRows; ++j) {
            const int r = base + j * ty;
            if (r >= r1) break;
            float xv[N], xd[N];
            V::unpack(rx[j], xv);
            V::unpack(rd[j], xd);
#pragma unroll
            for (int m = 0; m < NMIX; ++m) {
                float o[N];
#pragma unroll
                for (int e = 0; e < N; ++e) o[e] = with_mu ? qs_mix(mu[m][e], xv[e], xd[e]) : xd[e];
                *reinterpret_cast<uint4*>(q.out[m] + (size_t)r * rowb + (size_t)c0 * sizeof(IO)) = V::pack(o);
            }
        }
    }
}

// Scalar path for any C, group size and element-aligned pointers.
template <typename IO>
__global__ void __launch_bounds__(256) channel_mix_scalar_kernel(const ChannelMixParams p) {
    const long long n = (long long)p.BT * p.C;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long bt = idx / p.C;
        const int c = (int)(idx - bt * p.C);
        const int t = (int)(bt % p.T);
        const int h = t / p.W, w = t - h * p.W;
        const ShiftRule rule = shift_rule(c, p.g, p.ng, p.H, p.W, p.s);
        const float X = Io<IO>::ld1(p.x + idx * sizeof(IO));
        const float D = shift_ok(rule, h, w)
                            ? Io<IO>::ld1(p.x + (idx + (long long)rule.off * p.C) * sizeof(IO))
                            : 0.0f;
        const float dif = X - D;
        const float rr = p.mu_r ? fmaf(__ldg(p.mu_r + c), dif, D) : D;
        const float kk = p.mu_k ? fmaf(__ldg(p.mu_k + c), dif, D) : D;
        const float kp = fmaxf(kk, 0.0f);
        const float y = kp * kp * rcp(ex2(-rr * kLog2e) + 1.0f);
        Io<IO>::st1(p.out + idx * sizeof(IO), y);
    }
}

}  // namespace vrwkv
