// Shared device helpers of the sm_100a Vision-RWKV kernels: storage-type
// traits, packed float2 arithmetic and hardware transcendental instructions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace vrwkv {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// Packed float2 arithmetic.  On sm_100 these map to the paired FP32
// instructions, which retire two lanes of work per issue slot.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 max2(float2 a, float2 b) {
    return make_float2(fmaxf(a.x, b.x), fmaxf(a.y, b.y));
}

// Hardware base-2 exponential (MUFU.EX2, PTX ex2.approx.ftz.f32).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 ex2(float2 x) { return make_float2(ex2(x.x), ex2(x.y)); }

// 2^x with x capped at 126, so the result is finite.  Used for decay powers:
// a span that reaches past the end of the sequence (padding chunks) only ever
// multiplies zero aggregates, and a finite factor keeps 0 * factor == 0.
constexpr float kMaxExp2 = 126.0f;
__device__ __forceinline__ float ex2c(float x) { return ex2(fminf(x, kMaxExp2)); }
__device__ __forceinline__ float2 ex2c(float2 x) { return make_float2(ex2c(x.x), ex2c(x.y)); }
__device__ __forceinline__ float2 min2(float2 a, float2 b) {
    return make_float2(fminf(a.x, b.x), fminf(a.y, b.y));
}

// Hardware reciprocal (MUFU.RCP, PTX rcp.approx.ftz.f32).
__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 rcp(float2 x) { return make_float2(rcp(x.x), rcp(x.y)); }

// ---------------------------------------------------------------------------
// Storage-type traits.  A "pair" is two adjacent channels of one token.
// ---------------------------------------------------------------------------
template <typename IO>
struct Io;

template <>
struct Io<float> {
    static constexpr int kBytes = 4;
    __device__ __forceinline__ static float2 ld_pair(const char* p) {
        return *reinterpret_cast<const float2*>(p);
    }
    __device__ __forceinline__ static float ld1(const char* p) {
        return *reinterpret_cast<const float*>(p);
    }
    __device__ __forceinline__ static void st_pair(char* p, float2 v) {
        *reinterpret_cast<float2*>(p) = v;
    }
    __device__ __forceinline__ static void st1(char* p, float v) {
        *reinterpret_cast<float*>(p) = v;
    }
    __device__ __forceinline__ static float to_io(float v) { return v; }
};

template <>
struct Io<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    __device__ __forceinline__ static float2 ld_pair(const char* p) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    }
    __device__ __forceinline__ static float ld1(const char* p) {
        return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
    }
    __device__ __forceinline__ static void st_pair(char* p, float2 v) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __float22bfloat162_rn(v);
    }
    __device__ __forceinline__ static void st1(char* p, float v) {
        *reinterpret_cast<__nv_bfloat16*>(p) = __float2bfloat16_rn(v);
    }
    __device__ __forceinline__ static float to_io(float v) {
        return __bfloat162float(__float2bfloat16_rn(v));
    }
};

// ---------------------------------------------------------------------------
// Q-Shift source of one channel (eq. 9; q_shift listing).  The channel
// groups end at the listing's slice bounds b[j-1] = int(C*gamma*j), j = 1..4
// (C*gamma formed in double, times j, truncated; computed on the host):
// group j covers [b[j-1], b[j]) with b[-1] = 0, and channels >= b[3] are
// copied.  All-zero bounds make every channel a copy (no shift).  The group
// fixes a token offset and an admissible coordinate range: groups 0/1 test
// the column w, groups 2/3 the row h, group 4 always reads the token itself.
// ---------------------------------------------------------------------------
struct QsBounds {
    int b[4];
};

__host__ __device__ __forceinline__ int qs_group(int c, const QsBounds& g) {
    return (c >= g.b[0]) + (c >= g.b[1]) + (c >= g.b[2]) + (c >= g.b[3]);
}

struct ShiftRule {
    int off;      // token offset of the source
    int use_w;    // 1: test w, 0: test h
    int lo, hi;   // admissible [lo, hi) for the tested coordinate
};

// ng = number of shifted groups: 4 for Q-Shift (eq. 9), 2 for the
// bidirectional shift of sparse (MAE) inputs, whose vertical groups pass
// their channels through unchanged.
__device__ __forceinline__ ShiftRule shift_rule(int c, const QsBounds& g, int ng, int H, int W, int s) {
    int grp = qs_group(c, g);
    if (grp >= ng) grp = 4;
    ShiftRule r;
    switch (grp) {
    case 0: r = {-s, 1, s, W}; break;          // from w - s
    case 1: r = {s, 1, 0, W - s}; break;       // from w + s
    case 2: r = {-s * W, 0, s, H}; break;      // from h - s
    case 3: r = {s * W, 0, 0, H - s}; break;   // from h + s
    default: r = {0, 1, 0, 0x7fffffff}; break; // copied channel
    }
    return r;
}

__device__ __forceinline__ bool shift_ok(const ShiftRule& r, int h, int w) {
    int x = r.use_w ? w : h;
    return x >= r.lo && x < r.hi;
}

}  // namespace vrwkv
