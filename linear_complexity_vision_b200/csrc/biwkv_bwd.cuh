// Bi-WKV backward for sm_100a: gradients of eq. 5 ("Vision-RWKV Backbone",
// Linear Complexity Bidirectional Attention) with respect to k, v, w and u.
//
// For one (b, c) column, with p_i = e^{k_i - M}, a = e^{-w/T}, E = e^u and the
// two-sided decayed sum  S(x)_t = sum_{i != t} a^{|t-i|-1} x_i:
//
//   N = S(p v) + E p v,   D = S(p) + E p,   y = N / D        (eq. 5)
//   q = g / D,   r = q y                                     (g = dL/dy)
//   dL/dv = p (S(q) + E q)
//   dL/dk = v dL/dv - p (S(r) + E r)
//   dL/du = E sum_t p_t (q_t v_t - r_t)
//   dL/dw = -(1/T) sum_t (q_t H(p v)_t - r_t H(p)_t)
//
// where H(x)_t = sum_{i != t} (|t-i|-1) a^{|t-i|-1} x_i is the distance-
// weighted sum (S differentiated by w, times -T).  The factor e^{-M} cancels
// from every product, so M can be any common reference; the kernel uses the
// column maximum of k.
//
// S and H are two-sided linear scans.  In each direction a pair (A, H) is
// carried across a segment of L tokens whose own contribution is (a, h):
//   A' = a^L A + a,   H' = a^L (H + L A) + h,
// an associative composition, so both scans run as in the forward kernel:
// walks over a thread's 8 tokens, shuffle scans over the 8 chunks of a warp,
// a CTA scan over its 8 warps and an exchange across the CTAs of a cluster.
// Pass 1 scans (p v, p) with their H parts and yields y, q, r and the dw, du
// terms; pass 2 scans (q, r) and yields dk and dv.
//
// Work decomposition.  A CTA owns batch row b, a slab of 8 channels and 512
// tokens; T > 512 splits over a cluster of up to 8 CTAs (T <= 4096), which
// at two CTAs per SM spans four SMs and packs onto the GPCs far better than
// 16-CTA clusters.  Thread = 2 adjacent channels (packed float2) x 8
// consecutive tokens; the 32 lanes of a warp are 4 channel pairs x 8
// consecutive chunks; 256 threads, two CTAs per SM within 128 registers: the
// per-token forward states (pass 1) and prefix sums (pass 2) wait in shared
// memory between the two walks, and p v is recomputed from p and v instead of
// being kept.  Inputs of 16-byte-aligned tensors with C % 8 == 0 arrive by
// TMA in the forward kernel's tile layout (element stride 8 along T: sub-tile
// i, row q is token i of chunk q, so a warp's eight chunks read eight
// consecutive rows), into shared memory that the per-token stash reuses
// afterwards; other tensors load straight from global memory.
// The CTAs of a column exchange their records with asynchronous stores into
// each other's shared memory that complete on the receiver's mailbox
// mbarrier (one per exchange pass), so no cluster-wide barrier is waited on.
// Exponents are base 2 (log2 e is folded into k, u and w).
#pragma once

#include <cuda.h>

#include "biwkv_tma.cuh"
#include "common.cuh"

namespace vrwkv {
namespace bwd {

constexpr int kCS = 8;                     // channels per CTA (a column slab)
constexpr int kNP = kCS / 2;               // channel pairs
constexpr int kL = 8;                      // tokens per thread
constexpr int kThreads = 256;
constexpr int kNW = kThreads / 32;         // 8 warps
constexpr int kCPW = 32 / kNP;             // chunks per warp (8)
constexpr int kTc = kThreads / kNP * kL;   // 512 tokens per CTA
constexpr int kWarpTok = kCPW * kL;        // 64 tokens per warp
constexpr int kMaxT = 4096;
constexpr int kClusterMax = kMaxT / kTc;   // 8

struct alignas(64) Params {
    CUtensorMap map[3];  // k, v, g (TMA path)
    CUtensorMap omap[2]; // gk, gv in the same layout (TMA stores)
    unsigned int* err;   // device error word (bounded TMA wait)
    int tma;             // inputs arrive by TMA
    int tma_store;       // gk, gv leave by TMA stores from shared memory
    int imaj;            // tensor-memory kernel: map[] and omap[] are residue-major views (one box
                         // per tile; sub-tile i holds the tokens 8 m + i)
    const char* k;
    const char* v;
    const char* g;  // upstream gradient dL/dy
    const float* w;
    const float* u;
    char* gk;
    char* gv;
    float* gw;      // (B, C): per batch row
    float* gu;      // (B, C)
    int B, T, C;
    int Tc;         // tokens per CTA (kTc when the column spans several CTAs)
    int ncl;        // CTAs per column = cluster size
    int vec;        // channel-pair loads and stores allowed
    float invT;
};

// Pass-1 record of one channel pair: sums of p v and p with their
// distance-weighted parts.
struct alignas(16) R1 {
    float2 apv, ap, hpv, hp;
};
// Pass-2 record: sums of q and r.
struct alignas(16) R2 {
    float2 aq, ar;
};

__device__ __forceinline__ R1 r1_zero() { return {f2(0.f), f2(0.f), f2(0.f), f2(0.f)}; }
__device__ __forceinline__ R2 r2_zero() { return {f2(0.f), f2(0.f)}; }

// Carry `x` across a segment of L tokens (decay aL = a^L) and add the
// segment's own part `in`.
__device__ __forceinline__ R1 r1_cross(const R1& x, float2 aL, float L, const R1& in) {
    R1 o;
    o.apv = fma2(aL, x.apv, in.apv);
    o.ap = fma2(aL, x.ap, in.ap);
    o.hpv = fma2(aL, fma2(f2(L), x.apv, x.hpv), in.hpv);
    o.hp = fma2(aL, fma2(f2(L), x.ap, x.hp), in.hp);
    return o;
}
__device__ __forceinline__ R2 r2_cross(const R2& x, float2 aL, const R2& in) {
    return {fma2(aL, x.aq, in.aq), fma2(aL, x.ar, in.ar)};
}
__device__ __forceinline__ R1 r1_scale(const R1& x, float2 s) {
    return {mul2(s, x.apv), mul2(s, x.ap), mul2(s, x.hpv), mul2(s, x.hp)};
}

__device__ __forceinline__ float2 shfl_up2(float2 v, int d, int width) {
    return make_float2(__shfl_up_sync(0xffffffffu, v.x, d, width), __shfl_up_sync(0xffffffffu, v.y, d, width));
}
__device__ __forceinline__ float2 shfl_down2(float2 v, int d, int width) {
    return make_float2(__shfl_down_sync(0xffffffffu, v.x, d, width),
                       __shfl_down_sync(0xffffffffu, v.y, d, width));
}
__device__ __forceinline__ R1 shfl_up(const R1& x, int d, int width) {
    return {shfl_up2(x.apv, d, width), shfl_up2(x.ap, d, width), shfl_up2(x.hpv, d, width),
            shfl_up2(x.hp, d, width)};
}
__device__ __forceinline__ R1 shfl_down(const R1& x, int d, int width) {
    return {shfl_down2(x.apv, d, width), shfl_down2(x.ap, d, width), shfl_down2(x.hpv, d, width),
            shfl_down2(x.hp, d, width)};
}
__device__ __forceinline__ R2 shfl_up(const R2& x, int d, int width) {
    return {shfl_up2(x.aq, d, width), shfl_up2(x.ar, d, width)};
}
__device__ __forceinline__ R2 shfl_down(const R2& x, int d, int width) {
    return {shfl_down2(x.aq, d, width), shfl_down2(x.ar, d, width)};
}

// a^L for both channels of a pair: lam2 = w/T in base-2 units.
__device__ __forceinline__ float2 decay(float2 lam2, float L) {
    return ex2c(make_float2(-L * lam2.x, -L * lam2.y));
}

// Scalar component `hi` (0: .x, 1: .y) of a float2.
__device__ __forceinline__ float comp(float2 v, int hi) { return hi ? v.y : v.x; }
__device__ __forceinline__ void set_comp(float2& v, int hi, float x) {
    if (hi) v.y = x; else v.x = x;
}

struct alignas(16) Scratch {
    float2 wmax[kNW][kNP];       // per-warp maxima of k (base 2)
    // per-warp aggregates and exclusive carries, [pair][warp] with one element
    // of row padding against bank conflicts
    R1 w1F[kNP][kNW + 1], w1B[kNP][kNW + 1];
    R1 c1F[kNP][kNW + 1], c1B[kNP][kNW + 1];
    R2 w2F[kNP][kNW + 1], w2B[kNP][kNW + 1];
    R2 c2F[kNP][kNW + 1], c2B[kNP][kNW + 1];
    float2 wgw[kNW][kNP], wgu[kNW][kNP];  // per-warp dw, du partial sums
    // this CTA's records, staged for the pushes
    R1 own1F[kNP], own1B[kNP];
    float2 ownM[kNP];
    R2 own2F[kNP], own2B[kNP];
    float2 ownW[kNP], ownU[kNP];
    // mailboxes: each peer's records, written by the peers
    R1 mb1F[kClusterMax][kNP + 1], mb1B[kClusterMax][kNP + 1];
    float2 mbM[kClusterMax][kNP + 1];
    R2 mb2F[kClusterMax][kNP + 1], mb2B[kClusterMax][kNP + 1];
    float2 mbW[kClusterMax][kNP + 1], mbU[kClusterMax][kNP + 1];
    // carries into this CTA (common exponent Mc) and Mc itself
    R1 k1F[kNP], k1B[kNP];
    R2 k2F[kNP], k2B[kNP];
    float2 kMc[kNP];
    unsigned long long xbar[2];  // mailbox barriers of the two exchange passes
};

// Bytes one peer stores into a mailbox per channel pair: pass 1 two R1 and
// the maximum; pass 2 two R2, dw and du.
constexpr unsigned kRec1Bytes = 2 * sizeof(R1) + sizeof(float2);
constexpr unsigned kRec2Bytes = 2 * sizeof(R2) + 2 * sizeof(float2);

// Asynchronous store of one record into a peer's shared memory, completing
// its bytes on the peer's mailbox barrier.
__device__ __forceinline__ void st_async(unsigned raddr, const R1& x, unsigned rbar) {
    fast::st_async4(raddr, make_float4(x.apv.x, x.apv.y, x.ap.x, x.ap.y), rbar);
    fast::st_async4(raddr + 16, make_float4(x.hpv.x, x.hpv.y, x.hp.x, x.hp.y), rbar);
}
__device__ __forceinline__ void st_async(unsigned raddr, const R2& x, unsigned rbar) {
    fast::st_async4(raddr, make_float4(x.aq.x, x.aq.y, x.ar.x, x.ar.y), rbar);
}
__device__ __forceinline__ unsigned peer_addr(const void* local, int peer) {
    return fast::mapa_u32(fast::smem_u32(local), (unsigned)peer);
}

// Per-token state between the two walks of a pass, as two 16-byte planes
// [token][thread] (a thread's accesses are 16 bytes at a 16-byte stride:
// bank-conflict free): pass 1 keeps (apv, ap) in plane 0 and (hpv, hp) in
// plane 1; pass 2 keeps (aq, ar) in plane 0.
constexpr size_t kStashBytes = 2 * sizeof(float4) * kL * kThreads;
// the stash starts 128-byte aligned (it also receives the TMA tiles)
constexpr size_t kStashOff = (sizeof(Scratch) + 127) / 128 * 128;
constexpr size_t kSmemBytes = kStashOff + kStashBytes + 128;  // + re-alignment slack
constexpr int kTileRows = kTc / kL;  // rows of one sub-tile (64)

template <typename IO>
__device__ __forceinline__ float2 load_pair(const char* base, size_t row_elem, int cA, int C, bool ok_t,
                                            bool vec) {
    constexpr int es = Io<IO>::kBytes;
    if (!ok_t) return f2(0.0f);
    const char* p = base + (row_elem + cA) * es;
    if (vec && cA + 1 < C) return Io<IO>::ld_pair(p);
    return make_float2(cA < C ? Io<IO>::ld1(p) : 0.0f, cA + 1 < C ? Io<IO>::ld1(p + es) : 0.0f);
}

template <typename IO>
__device__ __forceinline__ void store_pair(char* base, size_t row_elem, int cA, int C, bool ok_t, bool vec,
                                           float2 val) {
    constexpr int es = Io<IO>::kBytes;
    if (!ok_t) return;
    char* p = base + (row_elem + cA) * es;
    if (vec && cA + 1 < C) {
        Io<IO>::st_pair(p, val);
    } else {
        if (cA < C) Io<IO>::st1(p, val.x);
        if (cA + 1 < C) Io<IO>::st1(p + es, val.y);
    }
}

template <typename IO>
__global__ void __launch_bounds__(kThreads, 2) biwkv_bwd_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(128) char smem_raw[];
    char* smem = smem_raw + ((128u - (fast::smem_u32(smem_raw) & 127u)) & 127u);
    Scratch& S = *reinterpret_cast<Scratch*>(smem);
    float4* plane0 = reinterpret_cast<float4*>(smem + kStashOff);  // [kL][kThreads]
    float4* plane1 = plane0 + kL * kThreads;
    __shared__ unsigned long long tma_bar;

    const int tid = threadIdx.x;
    const int j = tid % kNP;  // channel pair
    const int q = tid / kNP;  // chunk within the CTA (0..63)
    const int cq = q % kCPW;  // chunk within the warp
    const int warp = tid >> 5;
    const int rank = blockIdx.x;
    const int c0 = blockIdx.y * kCS;
    const int b = blockIdx.z;
    const int t0 = rank * p.Tc;
    const int tend = min(p.T, t0 + p.Tc);
    const int cA = c0 + 2 * j;
    const bool vec = p.vec != 0;
    const bool multi = p.ncl > 1;

    // ---- TMA: lanes 0..7 of warp 0 load sub-tile i of k, v and g --------------
    constexpr int es = Io<IO>::kBytes;
    constexpr int RB = kCS * es;           // bytes per token row of a tile
    constexpr int SUB = kTileRows * RB;    // bytes per sub-tile
    constexpr int TILE = kL * SUB;         // bytes per tile
    char* tiles = smem + kStashOff;        // k, v, g tiles (the stash later)
    if (tid == 0) {
        if (p.tma) fast::mbar_init(&tma_bar, 1);
        if (multi) {
            // mailbox barriers: one arrival (here) plus every peer's bytes
            fast::mbar_init(&S.xbar[0], 1);
            fast::mbar_expect_tx(&S.xbar[0], (unsigned)p.ncl * kNP * kRec1Bytes);
            fast::mbar_init(&S.xbar[1], 1);
            fast::mbar_expect_tx(&S.xbar[1], (unsigned)p.ncl * kNP * kRec2Bytes);
        }
    }
    __syncthreads();
    // every CTA's mailbox barriers exist before a peer stores: arrive now,
    // wait just before the first store
    if (multi) fast::cluster_arrive_relaxed();
    if (p.tma) {
        if (warp == 0) {
            if (tid == 0) fast::mbar_expect_tx(&tma_bar, (unsigned)(3 * TILE));
            __syncwarp();
            if (tid < kL) {
                // two boxes of 256 strided tokens (32 rows) per sub-tile
#pragma unroll
                for (int s3 = 0; s3 < 3; ++s3)
#pragma unroll
                    for (int h = 0; h < kTc / 256; ++h)
                        fast::tma_load_3d(tiles + s3 * TILE + tid * SUB + h * 32 * RB, &p.map[s3], c0,
                                          t0 + tid + 256 * h, b, &tma_bar);
            }
        }
    }

    // ---- per-channel constants -----------------------------------------------
    const float2 wv = make_float2(cA < p.C ? __ldg(p.w + cA) : 0.f, cA + 1 < p.C ? __ldg(p.w + cA + 1) : 0.f);
    const float2 uv = make_float2(cA < p.C ? __ldg(p.u + cA) : 0.f, cA + 1 < p.C ? __ldg(p.u + cA + 1) : 0.f);
    const float2 lam2 = mul2(wv, f2(p.invT * kLog2e));  // w/T, base 2
    const float2 alpha = decay(lam2, 1.0f);
    const float2 eu = ex2(mul2(uv, f2(kLog2e)));

    // ---- load k, v, g of the thread's 8 tokens -------------------------------
    const int s_tok = t0 + q * kL;
    float2 kk[kL], vv[kL], gg[kL];
    float2 mx = f2(-INFINITY);
    if (p.tma) {
        if (tid == 0) fast::mbar_wait_bounded(&tma_bar, p.err);
        __syncthreads();
        const int rowoff = q * RB + j * 2 * es;  // token i of chunk q: + i * SUB
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            const int o = rowoff + i * SUB;
            kk[i] = fast::lds_pair<IO>(tiles, o);
            vv[i] = fast::lds_pair<IO>(tiles + TILE, o);
            gg[i] = fast::lds_pair<IO>(tiles + 2 * TILE, o);
        }
    } else {
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            const int t = s_tok + i;
            const bool ok = t < tend;
            const size_t row = ((size_t)b * p.T + t) * p.C;
            kk[i] = load_pair<IO>(p.k, row, cA, p.C, ok, vec);
            vv[i] = load_pair<IO>(p.v, row, cA, p.C, ok, vec);
            gg[i] = load_pair<IO>(p.g, row, cA, p.C, ok, vec);
        }
    }
#pragma unroll
    for (int i = 0; i < kL; ++i) {
        // tokens past T: k = -inf makes p = 0; v and g are zero (TMA fill or
        // the masked loads), except stale tile rows, hence the explicit masks
        const bool ok = s_tok + i < tend;
        kk[i] = ok ? mul2(kk[i], f2(kLog2e)) : f2(-INFINITY);  // base 2; -inf => p = 0
        vv[i] = ok ? vv[i] : f2(0.0f);
        gg[i] = ok ? gg[i] : f2(0.0f);
        mx = max2(mx, kk[i]);
    }
    // CTA maximum of k per channel
#pragma unroll
    for (int d = kNP; d < 32; d <<= 1) {
        mx.x = fmaxf(mx.x, __shfl_xor_sync(0xffffffffu, mx.x, d));
        mx.y = fmaxf(mx.y, __shfl_xor_sync(0xffffffffu, mx.y, d));
    }
    if (cq == 0) S.wmax[warp][j] = mx;
    __syncthreads();
    float2 Mcta = S.wmax[0][j];
#pragma unroll
    for (int w = 1; w < kNW; ++w) Mcta = max2(Mcta, S.wmax[w][j]);
    // a column chunk may hold no token of a padded channel: keep M finite
    Mcta = make_float2(Mcta.x == -INFINITY ? 0.f : Mcta.x, Mcta.y == -INFINITY ? 0.f : Mcta.y);

    // ---- pass 1: p, thread-local sums (p v recomputed where needed) ----------
    float2 pp[kL];
#pragma unroll
    for (int i = 0; i < kL; ++i) pp[i] = ex2(add2(kk[i], make_float2(-Mcta.x, -Mcta.y)));
    R1 lf = r1_zero(), lb = r1_zero();
#pragma unroll
    for (int i = 0; i < kL; ++i) {  // forward: segment grows to the right
        lf.hpv = mul2(alpha, add2(lf.hpv, lf.apv));
        lf.hp = mul2(alpha, add2(lf.hp, lf.ap));
        lf.apv = fma2(alpha, lf.apv, mul2(pp[i], vv[i]));
        lf.ap = fma2(alpha, lf.ap, pp[i]);
    }
#pragma unroll
    for (int i = kL - 1; i >= 0; --i) {  // backward: segment grows to the left
        lb.hpv = mul2(alpha, add2(lb.hpv, lb.apv));
        lb.hp = mul2(alpha, add2(lb.hp, lb.ap));
        lb.apv = fma2(alpha, lb.apv, mul2(pp[i], vv[i]));
        lb.ap = fma2(alpha, lb.ap, pp[i]);
    }
    // warp scan over the kCPW chunks (lanes kNP apart)
    R1 fI = lf, bI = lb;
#pragma unroll
    for (int d = 1; d < kCPW; d <<= 1) {
        const float L = (float)(kL * d);
        const float2 aL = decay(lam2, L);
        const R1 o = shfl_up(fI, kNP * d, 32);
        if (cq >= d) fI = r1_cross(o, aL, L, fI);
        const R1 o2 = shfl_down(bI, kNP * d, 32);
        if (cq + d < kCPW) bI = r1_cross(o2, aL, L, bI);
    }
    R1 X1 = shfl_up(fI, kNP, 32), Y1 = shfl_down(bI, kNP, 32);  // lane-exclusive
    if (cq == 0) X1 = r1_zero();
    if (cq == kCPW - 1) Y1 = r1_zero();
    if (cq == kCPW - 1) S.w1F[j][warp] = fI;
    if (cq == 0) S.w1B[j][warp] = bI;
    __syncthreads();
    // CTA scan over the warps: thread (pair jj, warp wi)
    if (tid < kNP * kNW) {
        const int jj = tid / kNW, wi = tid % kNW;
        const float2 wjw = make_float2(c0 + 2 * jj < p.C ? __ldg(p.w + c0 + 2 * jj) : 0.f,
                                       c0 + 2 * jj + 1 < p.C ? __ldg(p.w + c0 + 2 * jj + 1) : 0.f);
        const float2 lj = mul2(wjw, f2(p.invT * kLog2e));
        R1 f = S.w1F[jj][wi], g = S.w1B[jj][wi];
#pragma unroll
        for (int d = 1; d < kNW; d <<= 1) {
            const float L = (float)(kWarpTok * d);
            const float2 aL = decay(lj, L);
            const R1 o = shfl_up(f, d, kNW);
            if (wi >= d) f = r1_cross(o, aL, L, f);
            const R1 o2 = shfl_down(g, d, kNW);
            if (wi + d < kNW) g = r1_cross(o2, aL, L, g);
        }
        R1 xw = shfl_up(f, 1, kNW), yw = shfl_down(g, 1, kNW);
        if (wi == 0) xw = r1_zero();
        if (wi == kNW - 1) yw = r1_zero();
        S.c1F[jj][wi] = xw;
        S.c1B[jj][wi] = yw;
        if (wi == kNW - 1) S.own1F[jj] = f;  // the CTA spans kTc tokens when multi
        if (wi == 0) {
            S.own1B[jj] = g;
            float2 M = S.wmax[0][jj];
            for (int w = 1; w < kNW; ++w) M = max2(M, S.wmax[w][jj]);
            S.ownM[jj] = make_float2(M.x == -INFINITY ? 0.f : M.x, M.y == -INFINITY ? 0.f : M.y);
        }
    }
    __syncthreads();
    // cluster exchange 1: asynchronous stores of the records into every
    // peer's mailbox (one (peer, pair, part) per thread), then a bounded wait
    // until this CTA's own mailbox is full
    if (multi) {
        fast::cluster_wait_acquire();  // every mailbox barrier is initialised
        for (int e = tid; e < p.ncl * kNP * 3; e += kThreads) {  // (peer, pair, part)
            const int peer = e / (kNP * 3), jj = (e / 3) % kNP, part = e % 3;
            const unsigned rbar = peer_addr(&S.xbar[0], peer);
            if (part == 0) st_async(peer_addr(&S.mb1F[rank][jj], peer), S.own1F[jj], rbar);
            else if (part == 1) st_async(peer_addr(&S.mb1B[rank][jj], peer), S.own1B[jj], rbar);
            else fast::st_async2(peer_addr(&S.mbM[rank][jj], peer), S.ownM[jj], rbar);
        }
        if (tid == 0) fast::mbar_wait_cluster_bounded(&S.xbar[0], p.err);
        __syncthreads();
    }
    // carries into this CTA: one thread per (channel, direction), a fixed-order
    // fold over the peers in the common exponent frame Mc
    if (tid < 2 * kCS) {
        const int lc = tid % kCS, dir = tid / kCS, jj = lc >> 1, hi = lc & 1;
        const float lw = (c0 + lc < p.C ? __ldg(p.w + c0 + lc) : 0.f) * (p.invT * kLog2e);
        float Mc = comp(S.ownM[jj], hi);
        float kapv = 0.f, kap = 0.f, khpv = 0.f, khp = 0.f;
        if (multi) {
            for (int r = 0; r < p.ncl; ++r) Mc = fmaxf(Mc, comp(S.mbM[r][jj], hi));
            const float aT = ex2c(-(float)p.Tc * lw), LT = (float)p.Tc;
            const int rs = dir == 0 ? 0 : p.ncl - 1, re = rank, st = dir == 0 ? 1 : -1;
            for (int r = rs; r != re; r += st) {
                const R1& m = dir == 0 ? S.mb1F[r][jj] : S.mb1B[r][jj];
                const float sc = ex2(comp(S.mbM[r][jj], hi) - Mc);
                khpv = aT * fmaf(LT, kapv, khpv) + sc * comp(m.hpv, hi);
                khp = aT * fmaf(LT, kap, khp) + sc * comp(m.hp, hi);
                kapv = fmaf(aT, kapv, sc * comp(m.apv, hi));
                kap = fmaf(aT, kap, sc * comp(m.ap, hi));
            }
        }
        R1& K = dir == 0 ? S.k1F[jj] : S.k1B[jj];
        set_comp(K.apv, hi, kapv);
        set_comp(K.ap, hi, kap);
        set_comp(K.hpv, hi, khpv);
        set_comp(K.hp, hi, khp);
        if (dir == 0) set_comp(S.kMc[jj], hi, Mc);
    }
    __syncthreads();

    // ---- pass 1: carries into the thread's chunk, then y, q, r ----------------
    const float2 Mc = S.kMc[j];
    const float2 sl = ex2(add2(Mcta, make_float2(-Mc.x, -Mc.y)));  // CTA frame -> common frame
    R1 KF, KB;
    {
        const float Lw = (float)(kWarpTok * warp), Ll = (float)(kL * cq);
        KF = r1_cross(S.k1F[j], decay(lam2, Lw), Lw, r1_scale(S.c1F[j][warp], sl));
        KF = r1_cross(KF, decay(lam2, Ll), Ll, r1_scale(X1, sl));
        const float Lw2 = (float)(kWarpTok * (kNW - 1 - warp)), Ll2 = (float)(kL * (kCPW - 1 - cq));
        KB = r1_cross(S.k1B[j], decay(lam2, Lw2), Lw2, r1_scale(S.c1B[j][warp], sl));
        KB = r1_cross(KB, decay(lam2, Ll2), Ll2, r1_scale(Y1, sl));
    }
#pragma unroll
    for (int i = 0; i < kL; ++i) pp[i] = mul2(pp[i], sl);  // p in the common frame
    // forward sums at each token (over the tokens before it), kept in the stash
#pragma unroll
    for (int i = 0; i < kL; ++i) {
        plane0[i * kThreads + tid] = make_float4(KF.apv.x, KF.apv.y, KF.ap.x, KF.ap.y);
        plane1[i * kThreads + tid] = make_float4(KF.hpv.x, KF.hpv.y, KF.hp.x, KF.hp.y);
        KF.hpv = mul2(alpha, add2(KF.hpv, KF.apv));
        KF.hp = mul2(alpha, add2(KF.hp, KF.ap));
        KF.apv = fma2(alpha, KF.apv, mul2(pp[i], vv[i]));
        KF.ap = fma2(alpha, KF.ap, pp[i]);
    }
    float2 qq[kL], rr[kL];
    float2 gwa = f2(0.f), gua = f2(0.f);
#pragma unroll
    for (int i = kL - 1; i >= 0; --i) {
        const float4 s0 = plane0[i * kThreads + tid], s1 = plane1[i * kThreads + tid];
        R1 fw;
        fw.apv = make_float2(s0.x, s0.y);
        fw.ap = make_float2(s0.z, s0.w);
        fw.hpv = make_float2(s1.x, s1.y);
        fw.hp = make_float2(s1.z, s1.w);
        const float2 pvi = mul2(pp[i], vv[i]);
        const float2 N = add2(add2(fw.apv, KB.apv), mul2(eu, pvi));
        const float2 D = add2(add2(fw.ap, KB.ap), mul2(eu, pp[i]));
        const float2 HN = add2(fw.hpv, KB.hpv);
        const float2 HD = add2(fw.hp, KB.hp);
        const float2 rD = rcp(D);
        const float2 y = mul2(N, rD);
        // Tokens past T (padding of the last CTA) take no part: their forward
        // sums are real sums carried over up to 255 positions, which can
        // overflow for w < 0, so they are selected away, not multiplied by 0.
        const bool real = s_tok + i < tend;
        qq[i] = real ? mul2(gg[i], rD) : f2(0.f);
        rr[i] = real ? mul2(qq[i], y) : f2(0.f);
        if (real) {
            gwa = add2(gwa, fma2(qq[i], HN, mul2(make_float2(-rr[i].x, -rr[i].y), HD)));
            gua = fma2(mul2(eu, pp[i]), fma2(qq[i], vv[i], make_float2(-rr[i].x, -rr[i].y)), gua);
        }
        KB.hpv = mul2(alpha, add2(KB.hpv, KB.apv));
        KB.hp = mul2(alpha, add2(KB.hp, KB.ap));
        KB.apv = fma2(alpha, KB.apv, pvi);
        KB.ap = fma2(alpha, KB.ap, pp[i]);
    }

    // ---- pass 2: sums of q and r ---------------------------------------------
    R2 mf = r2_zero(), mb = r2_zero();
#pragma unroll
    for (int i = 0; i < kL; ++i) {
        mf.aq = fma2(alpha, mf.aq, qq[i]);
        mf.ar = fma2(alpha, mf.ar, rr[i]);
    }
#pragma unroll
    for (int i = kL - 1; i >= 0; --i) {
        mb.aq = fma2(alpha, mb.aq, qq[i]);
        mb.ar = fma2(alpha, mb.ar, rr[i]);
    }
    R2 fJ = mf, bJ = mb;
#pragma unroll
    for (int d = 1; d < kCPW; d <<= 1) {
        const float2 aL = decay(lam2, (float)(kL * d));
        const R2 o = shfl_up(fJ, kNP * d, 32);
        if (cq >= d) fJ = r2_cross(o, aL, fJ);
        const R2 o2 = shfl_down(bJ, kNP * d, 32);
        if (cq + d < kCPW) bJ = r2_cross(o2, aL, bJ);
    }
    R2 X2 = shfl_up(fJ, kNP, 32), Y2 = shfl_down(bJ, kNP, 32);
    if (cq == 0) X2 = r2_zero();
    if (cq == kCPW - 1) Y2 = r2_zero();
    if (cq == kCPW - 1) S.w2F[j][warp] = fJ;
    if (cq == 0) S.w2B[j][warp] = bJ;
    // dw, du partial sums: over the warp's chunks, then over the warps
#pragma unroll
    for (int d = kNP; d < 32; d <<= 1) {
        gwa = add2(gwa, make_float2(__shfl_xor_sync(0xffffffffu, gwa.x, d), __shfl_xor_sync(0xffffffffu, gwa.y, d)));
        gua = add2(gua, make_float2(__shfl_xor_sync(0xffffffffu, gua.x, d), __shfl_xor_sync(0xffffffffu, gua.y, d)));
    }
    if (cq == 0) {
        S.wgw[warp][j] = gwa;
        S.wgu[warp][j] = gua;
    }
    __syncthreads();
    if (tid < kNP * kNW) {
        const int jj = tid / kNW, wi = tid % kNW;
        const float2 wjw = make_float2(c0 + 2 * jj < p.C ? __ldg(p.w + c0 + 2 * jj) : 0.f,
                                       c0 + 2 * jj + 1 < p.C ? __ldg(p.w + c0 + 2 * jj + 1) : 0.f);
        const float2 lj = mul2(wjw, f2(p.invT * kLog2e));
        R2 f = S.w2F[jj][wi], g = S.w2B[jj][wi];
#pragma unroll
        for (int d = 1; d < kNW; d <<= 1) {
            const float2 aL = decay(lj, (float)(kWarpTok * d));
            const R2 o = shfl_up(f, d, kNW);
            if (wi >= d) f = r2_cross(o, aL, f);
            const R2 o2 = shfl_down(g, d, kNW);
            if (wi + d < kNW) g = r2_cross(o2, aL, g);
        }
        R2 xw = shfl_up(f, 1, kNW), yw = shfl_down(g, 1, kNW);
        if (wi == 0) xw = r2_zero();
        if (wi == kNW - 1) yw = r2_zero();
        S.c2F[jj][wi] = xw;
        S.c2B[jj][wi] = yw;
        if (wi == kNW - 1) S.own2F[jj] = f;
        if (wi == 0) {
            S.own2B[jj] = g;
            float2 sw = S.wgw[0][jj], su = S.wgu[0][jj];
            for (int w = 1; w < kNW; ++w) {  // fixed order: deterministic
                sw = add2(sw, S.wgw[w][jj]);
                su = add2(su, S.wgu[w][jj]);
            }
            S.ownW[jj] = sw;
            S.ownU[jj] = su;
        }
    }
    __syncthreads();
    if (multi) {  // cluster exchange 2, as exchange 1 on the second mailbox barrier
        for (int e = tid; e < p.ncl * kNP * 4; e += kThreads) {  // (peer, pair, part)
            const int peer = e / (kNP * 4), jj = (e / 4) % kNP, part = e % 4;
            const unsigned rbar = peer_addr(&S.xbar[1], peer);
            if (part == 0) st_async(peer_addr(&S.mb2F[rank][jj], peer), S.own2F[jj], rbar);
            else if (part == 1) st_async(peer_addr(&S.mb2B[rank][jj], peer), S.own2B[jj], rbar);
            else if (part == 2) fast::st_async2(peer_addr(&S.mbW[rank][jj], peer), S.ownW[jj], rbar);
            else fast::st_async2(peer_addr(&S.mbU[rank][jj], peer), S.ownU[jj], rbar);
        }
        if (tid == 0) fast::mbar_wait_cluster_bounded(&S.xbar[1], p.err);
        __syncthreads();
    }
    if (tid < 2 * kCS) {
        const int lc = tid % kCS, dir = tid / kCS, jj = lc >> 1, hi = lc & 1;
        float kq = 0.f, kr = 0.f;
        if (multi) {
            const float lw = (c0 + lc < p.C ? __ldg(p.w + c0 + lc) : 0.f) * (p.invT * kLog2e);
            const float aT = ex2c(-(float)p.Tc * lw);
            const int rs = dir == 0 ? 0 : p.ncl - 1, re = rank, st = dir == 0 ? 1 : -1;
            for (int r = rs; r != re; r += st) {
                const R2& m = dir == 0 ? S.mb2F[r][jj] : S.mb2B[r][jj];
                kq = fmaf(aT, kq, comp(m.aq, hi));
                kr = fmaf(aT, kr, comp(m.ar, hi));
            }
        }
        R2& K = dir == 0 ? S.k2F[jj] : S.k2B[jj];
        set_comp(K.aq, hi, kq);
        set_comp(K.ar, hi, kr);
        // dw, du of the column: rank 0 folds the CTAs' partials in rank order
        if (rank == 0 && dir == 0 && c0 + lc < p.C) {
            float sw = comp(S.ownW[jj], hi), su = comp(S.ownU[jj], hi);
            if (multi) {
                sw = 0.f;
                su = 0.f;
                for (int r = 0; r < p.ncl; ++r) {
                    sw += comp(S.mbW[r][jj], hi);
                    su += comp(S.mbU[r][jj], hi);
                }
            }
            p.gw[(size_t)b * p.C + c0 + lc] = -sw * p.invT;
            p.gu[(size_t)b * p.C + c0 + lc] = su;
        }
    }
    __syncthreads();

    // ---- pass 2: carries, then dv and dk ------------------------------------------
    R2 QF, QB;
    {
        const float2 aW = decay(lam2, (float)(kWarpTok * warp)), aLn = decay(lam2, (float)(kL * cq));
        QF = r2_cross(r2_cross(S.k2F[j], aW, S.c2F[j][warp]), aLn, X2);
        const float2 aW2 = decay(lam2, (float)(kWarpTok * (kNW - 1 - warp)));
        const float2 aLn2 = decay(lam2, (float)(kL * (kCPW - 1 - cq)));
        QB = r2_cross(r2_cross(S.k2B[j], aW2, S.c2B[j][warp]), aLn2, Y2);
    }
#pragma unroll
    for (int i = 0; i < kL; ++i) {
        plane0[i * kThreads + tid] = make_float4(QF.aq.x, QF.aq.y, QF.ar.x, QF.ar.y);
        QF.aq = fma2(alpha, QF.aq, qq[i]);
        QF.ar = fma2(alpha, QF.ar, rr[i]);
    }
    // with TMA stores the results gather in two tiles in the stash's second
    // plane (free since pass 1), at the input tiles' offsets
    char* otile = reinterpret_cast<char*>(plane1);
    const int orow = q * RB + j * 2 * es;  // token i of chunk q: + i * SUB
#pragma unroll
    for (int i = kL - 1; i >= 0; --i) {
        const float4 s0 = plane0[i * kThreads + tid];
        R2 fq;
        fq.aq = make_float2(s0.x, s0.y);
        fq.ar = make_float2(s0.z, s0.w);
        const float2 Sq = fma2(eu, qq[i], add2(fq.aq, QB.aq));
        const float2 Sr = fma2(eu, rr[i], add2(fq.ar, QB.ar));
        const float2 dv = mul2(pp[i], Sq);
        const float2 dk = fma2(vv[i], dv, mul2(make_float2(-pp[i].x, -pp[i].y), Sr));
        if (p.tma_store) {
            Io<IO>::st_pair(otile + orow + i * SUB, dk);
            Io<IO>::st_pair(otile + TILE + orow + i * SUB, dv);
        } else {
            const int t = s_tok + i;
            const size_t row = ((size_t)b * p.T + t) * p.C;
            store_pair<IO>(p.gv, row, cA, p.C, t < tend, vec, dv);
            store_pair<IO>(p.gk, row, cA, p.C, t < tend, vec, dk);
        }
        QB.aq = fma2(alpha, QB.aq, qq[i]);
        QB.ar = fma2(alpha, QB.ar, rr[i]);
    }
    if (p.tma_store) {
        // lane i of warp 0 stores sub-tile i of gk and gv: boxes of 256
        // strided tokens, clipped at T by the tensor maps
        fast::fence_proxy_async_smem();
        __syncthreads();
        if (tid < kL) {
            const int nbox = (tend - t0 + 255) / 256;
#pragma unroll
            for (int o2 = 0; o2 < 2; ++o2)
                for (int hb = 0; hb < nbox; ++hb)
                    fast::tma_store_3d(&p.omap[o2], otile + o2 * TILE + tid * SUB + hb * 32 * RB, c0,
                                       t0 + tid + 256 * hb, b);
            fast::bulk_commit_and_wait_read();
        }
    }
    // no closing cluster barrier: every peer's stores into this CTA completed
    // before its second mailbox wait, and no CTA touches another's memory
    // after that
}

// dw, du of the batch: the per-row parts summed over b in order.
__global__ void __launch_bounds__(256) batch_sum_kernel(const float* in, float* out, int B, int C) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= C) return;
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += in[(size_t)b * C + c];
    out[c] = s;
}

}  // namespace bwd
}  // namespace vrwkv
