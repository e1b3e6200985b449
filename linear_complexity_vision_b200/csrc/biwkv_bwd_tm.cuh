// Bi-WKV backward for sm_100a with 16-token thread chunks whose per-token
// states live in tensor memory: gradients of eq. 5 ("Vision-RWKV Backbone",
// Linear Complexity Bidirectional Attention) with respect to k, v, w and u.
//
// The same two passes and scans as biwkv_bwd_kernel (biwkv_bwd.cuh, which
// states the formulas): pass 1 scans (p v, p) with their distance-weighted
// parts and yields y, q = g / D, r = q y and the dw, du terms; pass 2 scans
// (q, r) and yields dv = p (S(q) + E q) and dk = v dv - p (S(r) + E r).
//
// What changes: a thread owns a channel pair and 16 tokens (two halves of 8)
// instead of 8, so the warp, CTA and cluster scans of both passes, the two
// exchanges and the set-up are spread over twice the tokens; 128 threads
// (4 warps) cover the same 512-token CTA.  The state a thread carries
// between walks moves out of registers:
//  * p of its 16 tokens: a shared-memory stash [token][thread] (conflict-
//    free 8-byte accesses), written once;
//  * the pass-1 forward sums at each token of the current half (8 floats per
//    token) and q, r of all 16 tokens: the thread's lane of 128 tensor-memory
//    columns (tcgen05.st / tcgen05.ld), 64 for the states, 64 for q and r;
//  * k, v and g stay in the TMA tiles and are read again where needed.
// The pass-2 local sums of q and r are accumulated while pass 1 produces
// them (the forward one with explicit decay powers).  Results go into the
// dead k and g slots of the tiles (the same thread owns each slot) and
// leave by TMA stores.  Four CTAs per SM: their tensor memory fills the
// SM's 512 columns, and a shared-memory floor keeps a fifth CTA off.
#pragma once

#include "biwkv_bwd.cuh"
#include "biwkv_tm.cuh"

namespace vrwkv {
namespace bwd2 {

using bwd::R1;
using bwd::R2;
using bwd::r1_cross;
using bwd::r1_scale;
using bwd::r1_zero;
using bwd::r2_cross;
using bwd::r2_zero;
using bwd::decay;
using bwd::comp;
using bwd::set_comp;
using bwd::peer_addr;
using bwd::kRec1Bytes;
using bwd::kRec2Bytes;

constexpr int kCS = 8;                      // channels per CTA
constexpr int kNP = kCS / 2;                // channel pairs
constexpr int kThreads = 128;
constexpr int kNW = kThreads / 32;          // 4 warps
constexpr int kCPW = 32 / kNP;              // chunks per warp (8)
constexpr int kKL = 16;                     // tokens per thread
constexpr int kHL = 8;                      // tokens per half (= the TMA element stride)
constexpr int kTc = kThreads / kNP * kKL;   // 512 tokens per CTA
constexpr int kWarpTok = kCPW * kKL;        // 128 tokens per warp
constexpr int kClusterMax = 8;              // T <= 4096
constexpr int kTileRows = kTc / kHL;        // rows of one sub-tile (64)
constexpr int kTmemCols = 128;
constexpr int kColState = 0;                // 64 columns: pass-1 states of the current half
constexpr int kColQR = 64;                  // 64 columns: q, r of the 16 tokens
constexpr int kSmemFloor = 46 * 1024;       // at most four CTAs per SM

struct alignas(16) Scratch {
    float2 wmax[kNW][kNP];
    R1 w1F[kNP][kNW + 1], w1B[kNP][kNW + 1];
    R1 c1F[kNP][kNW + 1], c1B[kNP][kNW + 1];
    R2 w2F[kNP][kNW + 1], w2B[kNP][kNW + 1];
    R2 c2F[kNP][kNW + 1], c2B[kNP][kNW + 1];
    float2 wgw[kNW][kNP], wgu[kNW][kNP];
    R1 own1F[kNP], own1B[kNP];
    float2 ownM[kNP];
    R2 own2F[kNP], own2B[kNP];
    float2 ownW[kNP], ownU[kNP];
    R1 mb1F[kClusterMax][kNP + 1], mb1B[kClusterMax][kNP + 1];
    float2 mbM[kClusterMax][kNP + 1];
    R2 mb2F[kClusterMax][kNP + 1], mb2B[kClusterMax][kNP + 1];
    float2 mbW[kClusterMax][kNP + 1], mbU[kClusterMax][kNP + 1];
    R1 k1F[kNP], k1B[kNP];
    R2 k2F[kNP], k2B[kNP];
    float2 kMc[kNP];
    unsigned long long tma_bar;
    unsigned long long xbar[2];
    unsigned int tmem;
};

// Shared memory: the scratch block, then the three tiles (k, v, g; 128-byte
// aligned), then the p stash [16 tokens][128 threads] float2.
template <typename IO>
struct Layout {
    static constexpr int es = Io<IO>::kBytes;
    static constexpr int RB = kCS * es;           // bytes per token row
    static constexpr int SUB = kTileRows * RB;    // bytes per sub-tile
    static constexpr int TILE = kHL * SUB;        // bytes per tile (512 tokens)
    static constexpr size_t kTilesOff = (sizeof(Scratch) + 127) / 128 * 128;
    static constexpr size_t kStashOff = kTilesOff + 3 * (size_t)TILE;
    static constexpr size_t kBytes = kStashOff + sizeof(float2) * kKL * kThreads + 128;  // + alignment slack
};

__device__ __forceinline__ void tmem_st32(uint32_t a, const float (&v)[32]) { tm32::tmem_st32(a, v); }
__device__ __forceinline__ void tmem_ld32(uint32_t a, float (&v)[32]) { tm32::tmem_ld32(a, v); }

// Resident CTAs the register budget is cut for: four (bfloat16 tiles), three
// for float32 (its tiles allow no more).
template <typename IO>
constexpr int kMinCtas = sizeof(IO) == 2 ? 4 : 3;

template <typename IO>
__global__ void __launch_bounds__(kThreads, kMinCtas<IO>) biwkv_bwd_tm_kernel(const __grid_constant__ bwd::Params p) {
    using LY = Layout<IO>;
    constexpr int es = LY::es, RB = LY::RB, SUB = LY::SUB, TILE = LY::TILE;
    extern __shared__ __align__(128) char smem_raw[];
    char* smem = smem_raw + ((128u - (fast::smem_u32(smem_raw) & 127u)) & 127u);
    Scratch& S = *reinterpret_cast<Scratch*>(smem);
    char* tiles = smem + LY::kTilesOff;  // k, v, g; then dk in k's, dv in g's slots
    float2* pst = reinterpret_cast<float2*>(smem + LY::kStashOff);  // [token][thread]

    const int tid = threadIdx.x;
    const int j = tid % kNP;
    const int q = tid / kNP;     // chunk within the CTA (0..31)
    const int cq = q % kCPW;     // chunk within the warp
    const int warp = tid >> 5;
    const int rank = blockIdx.x;
    const int c0 = blockIdx.y * kCS;
    const int b = blockIdx.z;
    const int t0 = rank * p.Tc;
    const int tend = min(p.T, t0 + p.Tc);
    const int cA = c0 + 2 * j;
    const bool multi = p.ncl > 1;

    if (tid == 0) {
        fast::mbar_init(&S.tma_bar, 1);
        if (multi) {
            fast::mbar_init(&S.xbar[0], 1);
            fast::mbar_expect_tx(&S.xbar[0], (unsigned)p.ncl * kNP * kRec1Bytes);
            fast::mbar_init(&S.xbar[1], 1);
            fast::mbar_expect_tx(&S.xbar[1], (unsigned)p.ncl * kNP * kRec2Bytes);
        }
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         fast::smem_u32(&S.tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tm32::tc_fence_before();
    __syncthreads();
    tm32::tc_fence_after();
    if (multi) fast::cluster_arrive_relaxed();
    const uint32_t tmem = S.tmem + ((uint32_t)(warp * 32) << 16);

    // ---- TMA: each of k, v and g in one box from a residue-major view (token
    // 8 m + i at sub-tile i, row m), or lane i of warp 0 loads sub-tile i in
    // boxes of 256 strided tokens -------------------------------------------------
    if (warp == 0) {
        if (tid == 0) fast::mbar_expect_tx(&S.tma_bar, (unsigned)(3 * TILE));
        __syncwarp();
        if (p.imaj) {
            if (tid == 0) {
#pragma unroll
                for (int s3 = 0; s3 < 3; ++s3)
                    fast::tma_load_4d(tiles + s3 * TILE, &p.map[s3], c0, t0 / kHL, 0, b, &S.tma_bar);
            }
        } else if (tid < kHL) {
#pragma unroll
            for (int s3 = 0; s3 < 3; ++s3)
#pragma unroll
                for (int h = 0; h < kTc / 256; ++h)
                    fast::tma_load_3d(tiles + s3 * TILE + tid * SUB + h * 32 * RB, &p.map[s3], c0,
                                      t0 + tid + 256 * h, b, &S.tma_bar);
        }
    }

    const float2 wv = make_float2(__ldg(p.w + cA), __ldg(p.w + cA + 1));
    const float2 uv = make_float2(__ldg(p.u + cA), __ldg(p.u + cA + 1));
    const float2 lam2 = mul2(wv, f2(p.invT * kLog2e));  // w/T, base 2
    const float2 alpha = decay(lam2, 1.0f);
    const float2 a8 = decay(lam2, (float)kHL);
    const float2 eu = ex2(mul2(uv, f2(kLog2e)));
    float2 pw[kHL];  // a^i, i < 8
    pw[0] = f2(1.0f);
#pragma unroll
    for (int i = 1; i < kHL; ++i) pw[i] = min2(mul2(pw[i - 1], alpha), f2(0x1p126f));

    const int s_tok = t0 + q * kKL;  // the thread's first token
    // token 8 (2q + h) + i of the CTA: sub-tile i, row 2q + h
    auto off = [&](int h, int i) { return (2 * q + h) * RB + j * 2 * es + i * SUB; };
    auto ok_tok = [&](int h, int i) { return s_tok + h * kHL + i < tend; };

    if (tid == 0) fast::mbar_wait_bounded(&S.tma_bar, p.err);
    __syncthreads();

    // ---- CTA maximum of k (base 2) ---------------------------------------------
    float2 mx = f2(-INFINITY);
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < kHL; ++i) {
            const float2 k = mul2(fast::lds_pair<IO>(tiles, off(h, i)), f2(kLog2e));
            if (ok_tok(h, i)) mx = max2(mx, k);
        }
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
    Mcta = make_float2(Mcta.x == -INFINITY ? 0.f : Mcta.x, Mcta.y == -INFINITY ? 0.f : Mcta.y);

    // ---- pass 1: p (stashed), local sums of each half --------------------------
    R1 lf[2], lb[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float2 pp[kHL], vv[kHL];
#pragma unroll
        for (int i = 0; i < kHL; ++i) {
            const float2 k = fast::lds_pair<IO>(tiles, off(h, i));
            const float2 v = fast::lds_pair<IO>(tiles + TILE, off(h, i));
            const bool ok = ok_tok(h, i);
            pp[i] = ok ? ex2(fma2(k, f2(kLog2e), make_float2(-Mcta.x, -Mcta.y))) : f2(0.0f);
            vv[i] = ok ? v : f2(0.0f);
            pst[(h * kHL + i) * kThreads + tid] = pp[i];
        }
        R1 f = r1_zero(), g = r1_zero();
#pragma unroll
        for (int i = 0; i < kHL; ++i) {
            const int ib = kHL - 1 - i;
            f.hpv = mul2(alpha, add2(f.hpv, f.apv));
            f.hp = mul2(alpha, add2(f.hp, f.ap));
            f.apv = fma2(alpha, f.apv, mul2(pp[i], vv[i]));
            f.ap = fma2(alpha, f.ap, pp[i]);
            g.hpv = mul2(alpha, add2(g.hpv, g.apv));
            g.hp = mul2(alpha, add2(g.hp, g.ap));
            g.apv = fma2(alpha, g.apv, mul2(pp[ib], vv[ib]));
            g.ap = fma2(alpha, g.ap, pp[ib]);
        }
        lf[h] = f;
        lb[h] = g;
    }
    // the chunk's records: forward at its end, backward at its start
    R1 fI = r1_cross(lf[0], a8, (float)kHL, lf[1]);
    R1 bI = r1_cross(lb[1], a8, (float)kHL, lb[0]);
    // warp scan over the kCPW chunks (lanes kNP apart)
#pragma unroll
    for (int d = 1; d < kCPW; d <<= 1) {
        const float L = (float)(kKL * d);
        const float2 aL = decay(lam2, L);
        const R1 o = bwd::shfl_up(fI, kNP * d, 32);
        if (cq >= d) fI = r1_cross(o, aL, L, fI);
        const R1 o2 = bwd::shfl_down(bI, kNP * d, 32);
        if (cq + d < kCPW) bI = r1_cross(o2, aL, L, bI);
    }
    R1 X1 = bwd::shfl_up(fI, kNP, 32), Y1 = bwd::shfl_down(bI, kNP, 32);
    if (cq == 0) X1 = r1_zero();
    if (cq == kCPW - 1) Y1 = r1_zero();
    if (cq == kCPW - 1) S.w1F[j][warp] = fI;
    if (cq == 0) S.w1B[j][warp] = bI;
    __syncthreads();
    {
        // CTA scan, in every thread for its own pair (no warp waits for a
        // serial scan in warp 0): the exclusive carries into this thread's
        // warp, and the CTA's records from the lanes of chunk 0
        const float L = (float)kWarpTok;
        const float2 aW = decay(lam2, L);  // across one warp's tokens
        R1 acc = r1_zero(), xw = r1_zero();
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            if (w == warp) xw = acc;
            acc = r1_cross(acc, aW, L, S.w1F[j][w]);
        }
        R1 accb = r1_zero(), yw = r1_zero();
#pragma unroll
        for (int w = kNW - 1; w >= 0; --w) {
            if (w == warp) yw = accb;
            accb = r1_cross(accb, aW, L, S.w1B[j][w]);
        }
        if (cq == 0) {
            S.c1F[j][warp] = xw;
            S.c1B[j][warp] = yw;
        }
        if (tid < kNP) {  // warp 0, chunk 0: pair j = tid
            S.own1F[j] = acc;
            S.own1B[j] = accb;
            S.ownM[j] = Mcta;
        }
    }
    __syncthreads();
    if (multi) {
        fast::cluster_wait_acquire();  // every mailbox barrier is initialised
        for (int e = tid; e < p.ncl * kNP * 3; e += kThreads) {  // (peer, pair, part)
            const int peer = e / (kNP * 3), jj = (e / 3) % kNP, part = e % 3;
            const unsigned rbar = peer_addr(&S.xbar[0], peer);
            if (part == 0) bwd::st_async(peer_addr(&S.mb1F[rank][jj], peer), S.own1F[jj], rbar);
            else if (part == 1) bwd::st_async(peer_addr(&S.mb1B[rank][jj], peer), S.own1B[jj], rbar);
            else fast::st_async2(peer_addr(&S.mbM[rank][jj], peer), S.ownM[jj], rbar);
        }
        if (tid == 0) fast::mbar_wait_cluster_bounded(&S.xbar[0], p.err);
        __syncthreads();
    }
    if (tid < 2 * kCS) {
        const int lc = tid % kCS, dir = tid / kCS, jj = lc >> 1, hi = lc & 1;
        const float lw = __ldg(p.w + c0 + lc) * (p.invT * kLog2e);
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

    // ---- pass 1 output: carries into each half, then y, q, r -------------------------
    const float2 Mc = S.kMc[j];
    const float2 sl = ex2(add2(Mcta, make_float2(-Mc.x, -Mc.y)));  // CTA frame -> common frame
    R1 KF, KB;
    {
        const float Lw = (float)(kWarpTok * warp), Ll = (float)(kKL * cq);
        KF = r1_cross(S.k1F[j], decay(lam2, Lw), Lw, r1_scale(S.c1F[j][warp], sl));
        KF = r1_cross(KF, decay(lam2, Ll), Ll, r1_scale(X1, sl));
        const float Lw2 = (float)(kWarpTok * (kNW - 1 - warp)), Ll2 = (float)(kKL * (kCPW - 1 - cq));
        KB = r1_cross(S.k1B[j], decay(lam2, Lw2), Lw2, r1_scale(S.c1B[j][warp], sl));
        KB = r1_cross(KB, decay(lam2, Ll2), Ll2, r1_scale(Y1, sl));
    }
    // carries into the halves: forward into half 1 = the end state of half
    // 0's forward walk; backward into half 0 across half 1
    const R1 KB0 = r1_cross(KB, a8, (float)kHL, r1_scale(lb[1], sl));
    float2 gwa = f2(0.f), gua = f2(0.f);
    R2 mf[2], mb[2];  // pass-2 local sums of q and r per half
    R1 f = KF;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        // forward walk: the state before each token, four tokens per store
#pragma unroll
        for (int part = 0; part < 2; ++part) {
            float st[32];
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = part * 4 + ii;
                st[8 * ii + 0] = f.apv.x; st[8 * ii + 1] = f.apv.y;
                st[8 * ii + 2] = f.ap.x;  st[8 * ii + 3] = f.ap.y;
                st[8 * ii + 4] = f.hpv.x; st[8 * ii + 5] = f.hpv.y;
                st[8 * ii + 6] = f.hp.x;  st[8 * ii + 7] = f.hp.y;
                const float2 pi = mul2(pst[(h * kHL + i) * kThreads + tid], sl);
                const float2 vi = ok_tok(h, i) ? fast::lds_pair<IO>(tiles + TILE, off(h, i)) : f2(0.0f);
                f.hpv = mul2(alpha, add2(f.hpv, f.apv));
                f.hp = mul2(alpha, add2(f.hp, f.ap));
                f.apv = fma2(alpha, f.apv, mul2(pi, vi));
                f.ap = fma2(alpha, f.ap, pi);
            }
            tmem_st32(tmem + kColState + 32 * part, st);
        }
        tm32::tmem_wait_st();
        // backward walk: y, q, r and the dw, du terms; q, r are stashed and
        // summed both ways for pass 2
        R1 g = h == 0 ? KB0 : KB;
        R2 lmf = r2_zero(), lmb = r2_zero();
        float qr[32];  // per token i: q.x, q.y, r.x, r.y
#pragma unroll
        for (int part = 1; part >= 0; --part) {
            float st[32];
            tmem_ld32(tmem + kColState + 32 * part, st);
#pragma unroll
            for (int ii = 3; ii >= 0; --ii) {
                const int i = part * 4 + ii;
                const float2 fapv = make_float2(st[8 * ii + 0], st[8 * ii + 1]);
                const float2 fap = make_float2(st[8 * ii + 2], st[8 * ii + 3]);
                const float2 fhpv = make_float2(st[8 * ii + 4], st[8 * ii + 5]);
                const float2 fhp = make_float2(st[8 * ii + 6], st[8 * ii + 7]);
                const bool real = ok_tok(h, i);
                const float2 pi = mul2(pst[(h * kHL + i) * kThreads + tid], sl);
                const float2 vi = real ? fast::lds_pair<IO>(tiles + TILE, off(h, i)) : f2(0.0f);
                const float2 gi = real ? fast::lds_pair<IO>(tiles + 2 * TILE, off(h, i)) : f2(0.0f);
                const float2 pvi = mul2(pi, vi);
                const float2 N = add2(add2(fapv, g.apv), mul2(eu, pvi));
                const float2 D = add2(add2(fap, g.ap), mul2(eu, pi));
                const float2 HN = add2(fhpv, g.hpv);
                const float2 HD = add2(fhp, g.hp);
                const float2 rD = rcp(D);
                const float2 y = mul2(N, rD);
                // tokens past T take no part (their forward sums may overflow)
                const float2 qi = real ? mul2(gi, rD) : f2(0.f);
                const float2 ri = real ? mul2(qi, y) : f2(0.f);
                if (real) {
                    gwa = add2(gwa, fma2(qi, HN, mul2(make_float2(-ri.x, -ri.y), HD)));
                    gua = fma2(mul2(eu, pi), fma2(qi, vi, make_float2(-ri.x, -ri.y)), gua);
                }
                qr[4 * i + 0] = qi.x;
                qr[4 * i + 1] = qi.y;
                qr[4 * i + 2] = ri.x;
                qr[4 * i + 3] = ri.y;
                // pass-2 sums of the half: backward in walk order, forward
                // with the decay power to the half's last token
                lmb.aq = fma2(alpha, lmb.aq, qi);
                lmb.ar = fma2(alpha, lmb.ar, ri);
                lmf.aq = fma2(pw[kHL - 1 - i], qi, lmf.aq);
                lmf.ar = fma2(pw[kHL - 1 - i], ri, lmf.ar);
                g.hpv = mul2(alpha, add2(g.hpv, g.apv));
                g.hp = mul2(alpha, add2(g.hp, g.ap));
                g.apv = fma2(alpha, g.apv, pvi);
                g.ap = fma2(alpha, g.ap, pi);
            }
        }
        tmem_st32(tmem + kColQR + 32 * h, qr);
        mf[h] = lmf;
        mb[h] = lmb;
    }

    // ---- pass 2: sums of q and r ---------------------------------------------
    R2 fJ = r2_cross(mf[0], a8, mf[1]), bJ = r2_cross(mb[1], a8, mb[0]);
#pragma unroll
    for (int d = 1; d < kCPW; d <<= 1) {
        const float2 aL = decay(lam2, (float)(kKL * d));
        const R2 o = bwd::shfl_up(fJ, kNP * d, 32);
        if (cq >= d) fJ = r2_cross(o, aL, fJ);
        const R2 o2 = bwd::shfl_down(bJ, kNP * d, 32);
        if (cq + d < kCPW) bJ = r2_cross(o2, aL, bJ);
    }
    R2 X2 = bwd::shfl_up(fJ, kNP, 32), Y2 = bwd::shfl_down(bJ, kNP, 32);
    if (cq == 0) X2 = r2_zero();
    if (cq == kCPW - 1) Y2 = r2_zero();
    if (cq == kCPW - 1) S.w2F[j][warp] = fJ;
    if (cq == 0) S.w2B[j][warp] = bJ;
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
    {
        // CTA scan of pass 2, in every thread for its own pair as pass 1's
        const float2 aW = decay(lam2, (float)kWarpTok);
        R2 acc = r2_zero(), xw = r2_zero();
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            if (w == warp) xw = acc;
            acc = r2_cross(acc, aW, S.w2F[j][w]);
        }
        R2 accb = r2_zero(), yw = r2_zero();
#pragma unroll
        for (int w = kNW - 1; w >= 0; --w) {
            if (w == warp) yw = accb;
            accb = r2_cross(accb, aW, S.w2B[j][w]);
        }
        if (cq == 0) {
            S.c2F[j][warp] = xw;
            S.c2B[j][warp] = yw;
        }
        if (tid < kNP) {
            S.own2F[j] = acc;
            S.own2B[j] = accb;
            float2 sw = S.wgw[0][j], su = S.wgu[0][j];
            for (int w = 1; w < kNW; ++w) {  // fixed order: deterministic
                sw = add2(sw, S.wgw[w][j]);
                su = add2(su, S.wgu[w][j]);
            }
            S.ownW[j] = sw;
            S.ownU[j] = su;
        }
    }
    __syncthreads();
    if (multi) {
        for (int e = tid; e < p.ncl * kNP * 4; e += kThreads) {  // (peer, pair, part)
            const int peer = e / (kNP * 4), jj = (e / 4) % kNP, part = e % 4;
            const unsigned rbar = peer_addr(&S.xbar[1], peer);
            if (part == 0) bwd::st_async(peer_addr(&S.mb2F[rank][jj], peer), S.own2F[jj], rbar);
            else if (part == 1) bwd::st_async(peer_addr(&S.mb2B[rank][jj], peer), S.own2B[jj], rbar);
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
            const float lw = __ldg(p.w + c0 + lc) * (p.invT * kLog2e);
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
        if (rank == 0 && dir == 0) {
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

    // ---- pass 2 output: carries into each half, then dv and dk -------------------------
    R2 QF, QB;
    {
        const float2 aW = decay(lam2, (float)(kWarpTok * warp)), aLn = decay(lam2, (float)(kKL * cq));
        QF = r2_cross(r2_cross(S.k2F[j], aW, S.c2F[j][warp]), aLn, X2);
        const float2 aW2 = decay(lam2, (float)(kWarpTok * (kNW - 1 - warp)));
        const float2 aLn2 = decay(lam2, (float)(kKL * (kCPW - 1 - cq)));
        QB = r2_cross(r2_cross(S.k2B[j], aW2, S.c2B[j][warp]), aLn2, Y2);
    }
    const R2 QB0 = r2_cross(QB, a8, mb[1]);
    tm32::tmem_wait_st();  // q and r are in tensor memory
    char* tk = tiles;             // dk into k's slots (k is dead: p is stashed)
    char* tg = tiles + 2 * TILE;  // dv into g's slots (g is dead after pass 1)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float qr[32];
        tmem_ld32(tmem + kColQR + 32 * h, qr);
        float2 fq[kHL], fr[kHL];  // forward sums before each token
#pragma unroll
        for (int i = 0; i < kHL; ++i) {
            fq[i] = QF.aq;
            fr[i] = QF.ar;
            QF.aq = fma2(alpha, QF.aq, make_float2(qr[4 * i], qr[4 * i + 1]));
            QF.ar = fma2(alpha, QF.ar, make_float2(qr[4 * i + 2], qr[4 * i + 3]));
        }
        // (QF now carries into the next half)
        R2 g = h == 0 ? QB0 : QB;
#pragma unroll
        for (int i = kHL - 1; i >= 0; --i) {
            const float2 qi = make_float2(qr[4 * i], qr[4 * i + 1]), ri = make_float2(qr[4 * i + 2], qr[4 * i + 3]);
            const float2 pi = mul2(pst[(h * kHL + i) * kThreads + tid], sl);
            const float2 vi = fast::lds_pair<IO>(tiles + TILE, off(h, i));
            const float2 Sq = fma2(eu, qi, add2(fq[i], g.aq));
            const float2 Sr = fma2(eu, ri, add2(fr[i], g.ar));
            const float2 dv = mul2(pi, Sq);
            const float2 dk = fma2(vi, dv, mul2(make_float2(-pi.x, -pi.y), Sr));
            Io<IO>::st_pair(tk + off(h, i), dk);
            Io<IO>::st_pair(tg + off(h, i), dv);
            g.aq = fma2(alpha, g.aq, qi);
            g.ar = fma2(alpha, g.ar, ri);
        }
    }
    // lane i of warp 0 stores sub-tile i of dk and dv: boxes of 256 strided
    // tokens, clipped at T by the tensor maps
    fast::fence_proxy_async_smem();
    tm32::tc_fence_before();
    __syncthreads();
    if (tid < kHL) {
        if (p.imaj) {
            if (tid == 0) {
                fast::tma_store_4d(&p.omap[0], tk, c0, t0 / kHL, 0, b);
                fast::tma_store_4d(&p.omap[1], tg, c0, t0 / kHL, 0, b);
            }
        } else {
            const int nbox = (tend - t0 + 255) / 256;
            for (int hb = 0; hb < nbox; ++hb) {
                fast::tma_store_3d(&p.omap[0], tk + tid * SUB + hb * 32 * RB, c0, t0 + tid + 256 * hb, b);
                fast::tma_store_3d(&p.omap[1], tg + tid * SUB + hb * 32 * RB, c0, t0 + tid + 256 * hb, b);
            }
        }
        fast::bulk_commit_and_wait_read();
    }
    if (warp == 1) {
        tm32::tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(S.tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace bwd2
}  // namespace vrwkv
