// Fused Q-Shift -> Bi-WKV -> sigma(R) gate with 32-token thread chunks whose
// per-token partial sums live in tensor memory (sm_100a).
//
// Evaluates Bi-WKV of "Vision-RWKV Backbone", Linear Complexity
// Bidirectional Attention, eq. 5, on inputs Q-Shifted per Quad-Directional
// Token Shift, eq. 9, gated per Overall Architecture, eq. 2 -- the same
// chunked two-sided scan as the 8-channel TMA kernel (biwkv_tma.cuh):
//
//   A_t = sum_{i<t} a^{t-1-i} p_i v_i,  B_t = sum_{i>t} a^{i-t-1} p_i v_i,
//   C_t, D_t with v = 1,  a = e^{-w/T},  p_i = e^{k_i - M},
//   wkv_t = (A_t + B_t + e^u p_t v_t) / (C_t + D_t + e^u p_t).
//
// What changes against that kernel: a thread owns a channel pair and 32
// tokens (four sub-chunks of 8) instead of 16, so the fixed per-thread cost
// of the warp, CTA and cluster scans, the exchange and the set-up is spread
// over twice the tokens.  The 128 per-token partial sums a thread carries
// from the local pass to the output pass (numerator and denominator of 32
// tokens x 2 channels) do not fit next to the scan state in registers; they
// go to the thread's own lane of tensor memory (tcgen05.st, 32 columns per
// sub-chunk) and come back one sub-chunk at a time (tcgen05.ld).  A CTA holds
// 128 columns, so four CTAs fill an SM's 512; the host keeps at most four
// resident (a shared-memory floor) so an allocation never waits.
//
// The gate factor e^{-r} of a token is parked in two tile slots the thread
// has just read (r's own and shifted r's; without Q-Shift, r's and k's, or
// r's and one extra tile when one x feeds r, k and v), so no shared-memory
// array of gate factors is needed; the result later goes into the first
// slot.  Every slot is read and written by the one thread that owns the
// token.
//
// A CTA covers 1024 tokens x 8 channels; longer columns use a cluster of up
// to 8 CTAs along T (T <= 8192) exchanging their aggregates through
// asynchronous shared-memory stores, as in the 8-channel kernel.
//
// Copies: the TMA's cost grows with the number of boxes, so where T is a
// multiple of 8 a whole tile arrives in one box from a residue-major view
// (token 8 m + i lands at sub-tile i, row m) and the CTA's results leave in
// one store; elsewhere lane i of warp 0 moves sub-tile i in lane-strided
// boxes.  Q-Shift reads the image view where W allows and the flat token
// view otherwise (see the loads below).
#pragma once

#include "biwkv_tma.cuh"

namespace vrwkv {
namespace tm32 {

using fast::kCS;
using fast::kKV;
using fast::kL;
using fast::kNP;
using fast::kRKV;
using fast::kX;
using fast::bulk_commit_and_wait_read;
using fast::cluster_arrive_relaxed;
using fast::cluster_wait_acquire;
using fast::fence_proxy_async_smem;
using fast::fma4;
using fast::hi2;
using fast::lds_f32;
using fast::lds_pair;
using fast::lo2;
using fast::mapa_u32;
using fast::mbar_expect_tx;
using fast::mbar_init;
using fast::mbar_wait_bounded;
using fast::mbar_wait_cluster_bounded;
using fast::shfl_down4;
using fast::shfl_up4;
using fast::smem_u32;
using fast::st_async2;
using fast::st_async4;
using fast::sts_f32;
using fast::tma_load_3d;
using fast::tma_load_4d;
using fast::tma_load_5d;
using fast::tma_store_3d;
using fast::zero4;

constexpr int kThreads = 128;              // 4 channel pairs x 32 chunks
constexpr int kKL = 32;                    // tokens per thread chunk
constexpr int kH = kKL / kL;               // sub-chunks of 8 per chunk
constexpr int kNW = kThreads / 32;         // warps
constexpr int kCPW = 32 / kNP;             // chunks per warp
constexpr int kTc = kThreads / kNP * kKL;  // tokens per CTA (1024)
constexpr int kChunks = kTc / kKL;         // chunks per CTA
constexpr int kWarpTok = kCPW * kKL;       // tokens per warp (256)
constexpr int kClusterMax = 8;             // CTAs per column: T <= 8192
constexpr int kTmemCols = kH * 32;         // num, den of 32 tokens x 2 channels
// Dynamic shared memory of at least this many bytes keeps five CTAs from
// fitting on an SM (228 KB, 1 KB reserved per CTA): at most four CTAs hold
// tensor memory at once, 4 x 128 = 512 columns.
constexpr int kSmemFloor = 46 * 1024;

struct alignas(16) Scratch {
    float2 tab[kChunks][kNP];  // a^(32 m) per channel pair
    float2 wmax[kNP][kNW + 1];
    float4 waggF[kNP][kNW + 1];
    float4 waggB[kNP][kNW + 1];
    float2 mbM[kClusterMax][kNP + 1];
    float4 mbF[kClusterMax][kNP + 1];
    float4 mbG[kClusterMax][kNP + 1];
    float4 ownF[kNP];
    float4 ownG[kNP];
    float2 ownM[kNP];
    unsigned long long bar[kNW];  // tile boxes of warp w's 256 tokens
    unsigned long long xbar;
    unsigned int tmem;  // base address of this CTA's tensor-memory columns
    int tk;             // GX: this CTA's ticket
    unsigned int gen;   // GX: the launch's generation
};

// Per-thread sub-chunk values in natural sub-chunk order, for the rotated
// kernel: entry [h][thread] (threads fastest: conflict-free 16-byte
// accesses).  Holds the sub-chunk totals after the load pass, then the
// carries into each sub-chunk for the output pass.
struct alignas(16) Stash {
    float4 a[kH][kThreads];  // totals F_h (A.xy, C.xy), then carries from the left
    float4 b[kH][kThreads];  // totals G_h, then carries from the right
};

// 32 consecutive 32-bit columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]),
        "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15]), "f"(v[16]),
        "f"(v[17]), "f"(v[18]), "f"(v[19]), "f"(v[20]), "f"(v[21]), "f"(v[22]), "f"(v[23]), "f"(v[24]),
        "f"(v[25]), "f"(v[26]), "f"(v[27]), "f"(v[28]), "f"(v[29]), "f"(v[30]), "f"(v[31])
        : "memory");
}
// Load and wait in one statement, so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]),
          "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]), "=f"(v[19]), "=f"(v[20]), "=f"(v[21]),
          "=f"(v[22]), "=f"(v[23]), "=f"(v[24]), "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]),
          "=f"(v[29]), "=f"(v[30]), "=f"(v[31])
        : "r"(taddr)
        : "memory");
}
// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ROT: lanes take their four sub-chunks in a rotated order (lane pair m of
// a warp starts at sub-chunk m), so at every step the warp's 32 lanes touch
// 8 different 16-byte rows of each 128-byte line: conflict-free tile, gate
// and result accesses for 16-byte token rows.  The sub-chunk values that are
// needed in natural order pass through a per-thread stash.
// GX: no cluster; the CTAs of a column take tickets from the caller's
// workspace and exchange their records through it (the 8-channel kernel's
// workspace format and protocol: biwkv_tma.cuh).
template <typename IO, int LAYOUT, bool QS, bool ROT, bool GX>
__global__ void __launch_bounds__(kThreads, 4) biwkv_tm_kernel(const __grid_constant__ fast::Params p) {
    constexpr bool GATE = LAYOUT != kKV;
    constexpr int NSRC = LAYOUT == kKV ? 2 : (LAYOUT == kRKV ? 3 : 1);
    constexpr int NTILE = NSRC * (QS ? 2 : 1);
    constexpr int SR = 0;
    constexpr int SK = LAYOUT == kRKV ? 1 : 0;
    constexpr int SV = LAYOUT == kKV ? 1 : (LAYOUT == kRKV ? 2 : 0);
    constexpr int es = Io<IO>::kBytes;
    constexpr int RB = kCS * es;         // bytes per token row of a tile
    constexpr int PB = 2 * es;           // bytes per channel pair
    constexpr int SUB = kTc / kL * RB;   // bytes per sub-tile (128 token rows)

    extern __shared__ __align__(128) char smem_raw[];
    char* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    // The gate factor's two halves are parked in r's slot and, with Q-Shift,
    // in shifted r's slot (both read to make r); without Q-Shift in k's slot
    // (separate r, k, v) or in one extra tile (one x), so no slot another
    // value still needs is overwritten.
    constexpr bool G1_IN_K = GATE && !QS && LAYOUT == kRKV;
    constexpr int NTA = GATE && !QS && !G1_IN_K ? NTILE + 1 : NTILE;
    constexpr int G1 = QS ? 2 * SR + 1 : (G1_IN_K ? SK : NTILE);  // tile of the second half
    Scratch& S = *reinterpret_cast<Scratch*>(smem + NTA * p.tile_bytes);
    Stash& X2 = *reinterpret_cast<Stash*>(smem + NTA * p.tile_bytes + sizeof(Scratch));  // ROT only

    const int tid = threadIdx.x;
    const int j = tid % kNP;   // channel pair
    const int q = tid / kNP;   // chunk within the CTA
    const int cq = q % kCPW;   // chunk within the warp
    const int warp = tid >> 5;
    if (tid == 0) {
#pragma unroll
        for (int w = 0; w < kNW; ++w) mbar_init(&S.bar[w], 1);
        if (!GX && p.ncl > 1) {
            mbar_init(&S.xbar, 1);
            mbar_expect_tx(&S.xbar, (unsigned)(p.ncl * kNP * (sizeof(float4) * 2 + sizeof(float2))));
        }
        if (GX) {
            S.tk = (int)atomicAdd(p.ws_ctl, 1u);
            S.gen = *reinterpret_cast<volatile unsigned int*>(p.ws_ctl + 2);
        }
    }
    if (GX) {
        // a ticket outside the grid means a workspace that was not zero-filled:
        // leave before any tensor memory is taken
        __syncthreads();
        if (S.tk < 0 || S.tk >= p.total) {
            if (tid == 0) atomicOr(p.err, 4u);
            return;
        }
    }

    // this CTA's column chunk: the block index, or (GX) the ticket, column by
    // column so a column's CTAs hold consecutive tickets
    int rank = blockIdx.x, slab = blockIdx.y, b = blockIdx.z;
    unsigned int gen = 0;
    if (GX) {
        const int t = S.tk;
        gen = S.gen;
        rank = t % p.ncl;
        slab = (t / p.ncl) % p.nslab;
        b = t / p.ncl / p.nslab;
    }
    const int col = b * p.nslab + slab;  // GX: the column's records and flags
    const int c0 = slab * kCS;
    const int t0 = rank * p.Tc;
    const int tend = min(p.T, t0 + p.Tc);
    int grp = QS ? qs_group(c0, p.g) : 4;
    if (grp >= p.ng) grp = 4;
    const bool shifted = QS && grp < 4;

    // ---- tile loads, first of all.  Fewer, larger boxes cost the TMA less per
    // byte (measured), so where the shape allows (imaj) a tile arrives in one
    // box from a residue-major view that puts token 8 m + i at sub-tile i, row
    // m: (C, T / 8, 8, B) over the flat tokens, (C, W / 8, H, 8, B) over the
    // image with Q-Shift.  A vertical shift displaces the image box along h; a
    // horizontal shift (and any shift in the flat view) has lane i of warp 0
    // load sub-tile i of the shifted tile from a lane-strided view (xmap):
    // displaced by +-s along w in the image, by the group's token offset in
    // the flat tokens.  Elsewhere lane i loads sub-tile i of every tile in
    // nbox boxes; box g holds the tokens of warps g * 4 / nbox onwards and
    // completes on tile barrier g. ----------------------------------------------------
    const bool img = QS && !p.flat;
    const int nb = p.nbox, wpb = kNW / nb;  // boxes per lane and tile, warps per box
    if (warp == 0) {
        const int dw = grp == 0 ? -p.s : (grp == 1 ? p.s : 0);
        const int dh = grp == 2 ? -p.s : (grp == 3 ? p.s : 0);
        const int dt = dw + dh * p.W;
        const int r0 = rank * p.rows;
        if (p.imaj) {
            if (tid == 0) mbar_expect_tx(&S.bar[0], (unsigned)p.tile_bytes * (unsigned)(NSRC * (shifted ? 2 : 1)));
            __syncwarp();
            const bool one_shift = img && dh != 0;  // the shifted tile in one box too
            for (int s = 0; s < NSRC; ++s) {
                char* tile = smem + (QS ? 2 * s : s) * p.tile_bytes;
                if (tid == 0) {
                    if (img) {
                        tma_load_5d(tile, &p.map[s], c0, 0, r0, 0, b, &S.bar[0]);
                        if (shifted && one_shift) tma_load_5d(tile + p.tile_bytes, &p.map[s], c0, 0, r0 + dh, 0, b, &S.bar[0]);
                    } else {
                        tma_load_4d(tile, &p.map[s], c0, t0 / kL, 0, b, &S.bar[0]);
                    }
                }
                if (shifted && !one_shift && tid < kL) {
                    char* sh = tile + p.tile_bytes + tid * SUB;
                    if (img) {
                        tma_load_4d(sh, &p.xmap[s], c0, tid + dw, r0, b, &S.bar[0]);
                    } else {
#pragma unroll
                        for (int g = 0; g < kNW; ++g)
                            tma_load_3d(sh + g * 32 * RB, &p.xmap[s], c0, t0 + tid + dt + 256 * g, b, &S.bar[0]);
                    }
                }
            }
        } else {
            // bytes per lane and source: p.box_bytes in all, a share per box
            const unsigned copies = (unsigned)(kL * NSRC * (shifted ? 2 : 1));
            if (tid < nb) mbar_expect_tx(&S.bar[tid], (unsigned)p.box_bytes / (unsigned)nb * copies);
            __syncwarp();
            if (tid < kL) {
                const int i = tid;
                for (int g = 0; g < nb; ++g) {
                    for (int s = 0; s < NSRC; ++s) {
                        char* plain = smem + (QS ? 2 * s : s) * p.tile_bytes + i * SUB + g * wpb * 32 * RB;
                        if (img) {
                            tma_load_4d(plain, &p.map[s], c0, i, r0, b, &S.bar[g]);
                            if (shifted) tma_load_4d(plain + p.tile_bytes, &p.map[s], c0, i + dw, r0 + dh, b, &S.bar[g]);
                        } else {
                            tma_load_3d(plain, &p.map[s], c0, t0 + i + 256 * g, b, &S.bar[g]);
                            if (QS && shifted)
                                tma_load_3d(plain + p.tile_bytes, &p.map[s], c0, t0 + i + dt + 256 * g, b, &S.bar[g]);
                        }
                    }
                }
            }
        }
    }

    // ---- per-thread constants (overlap the copies) -------------------------------
    const int cA = c0 + 2 * j;
    const float invT = p.invT;
    const float2 wv = make_float2(__ldg(p.w + cA), __ldg(p.w + cA + 1));
    const float2 uv = make_float2(__ldg(p.u + cA), __ldg(p.u + cA + 1));
    const float2 lam2 = mul2(wv, f2(invT * kLog2e));  // w / T in base-2 units
    const float2 alpha = ex2c(make_float2(-lam2.x, -lam2.y));
    const float2 eu = ex2(mul2(uv, f2(kLog2e)));
    const float2 a8 = ex2c(mul2(lam2, f2(-(float)kL)));  // a^8: across one sub-chunk
    auto mu_of = [&](const float* m) { return m ? make_float2(__ldg(m + cA), __ldg(m + cA + 1)) : f2(0.0f); };
    const float2 muk = QS ? mu_of(p.mu[1]) : f2(1.0f);
    const float2 muv = QS ? mu_of(p.mu[2]) : f2(1.0f);
    const float2 mur = (QS && GATE) ? mu_of(p.mu[0]) : f2(1.0f);
    S.tab[q][j] = ex2c(mul2(lam2, f2(-(float)kKL * q)));  // a^(32 q)

    const int nvt = max(0, min(kKL, tend - (t0 + q * kKL)));  // valid tokens of this chunk

    // tensor memory; the CTA barrier also publishes the decay table and the
    // tile barriers' initialisation to every warp
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&S.tmem)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (!GX && p.ncl > 1) cluster_arrive_relaxed();  // waited for before the first push
    // this thread's lane of the CTA's columns
    const uint32_t tmem = S.tmem + ((uint32_t)(warp * 32) << 16);

    // this warp's tokens: with a barrier per warp every lane waits (bounded)
    // for its boxes; with Q-Shift in a horizontal group the warp then clears
    // its row-wrapped tokens of the shifted tiles
    if (nb == 1) {
        // one barrier: one thread waits, the others sleep at the CTA barrier
        if (tid == 0) mbar_wait_bounded(&S.bar[0], p.err);
        __syncthreads();
    } else {
        mbar_wait_bounded(&S.bar[warp / wpb], p.err);
    }
    if (QS && p.flat && shifted && grp < 2) {
        const int lo = t0 + warp * kWarpTok;
        fast::zero_row_wrap<RB>(smem, p.tile_bytes, SUB, NSRC, t0, lo, min(tend, lo + kWarpTok), p.W, p.s,
                                grp == 0, tid & 31, 32);
        __syncwarp();
    }

    // ---- 1-2. per 8-token sub-chunk: load, Q-Shift mix, gate factor (parked in
    // the token's slots), local maximum, p = 2^(k - M_h), two-sided sums inside
    // the sub-chunk; the per-token sums go to tensor memory -------------------------
    const char* tK = smem + (QS ? 2 * SK : SK) * p.tile_bytes;
    const char* tV = smem + (QS ? 2 * SV : SV) * p.tile_bytes;
    const char* tR = smem + (QS ? 2 * SR : SR) * p.tile_bytes;
    const int dsh = shifted ? p.tile_bytes : 0;
    char* g0 = smem + (QS ? 2 * SR : SR) * p.tile_bytes;  // gate factor, first channel
    char* g1 = smem + G1 * p.tile_bytes;                 // second channel
    const int rot = ROT ? (cq >> 1) & (kH - 1) : 0;
    float4 Fh[kH], Gh[kH];  // by step: the totals of sub-chunk (step + rot) mod 4
    float2 Mh[kH];
#pragma unroll
    for (int st = 0; st < kH; ++st) {
        const int h = ROT ? (st + rot) & (kH - 1) : st;  // the sub-chunk of this step
        const int rowoff = (q * kH + h) * RB + j * PB;
        const int nv = max(0, min(kL, nvt - h * kL));
        float2 kk[kL], vv[kL];
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            const int o = rowoff + i * SUB;
            float2 k, v, r;
            if (QS) {
                if (LAYOUT == kX) {
                    const float2 x = lds_pair<IO>(tK, o), xd = lds_pair<IO>(tK + dsh, o);
                    const float2 d = fma2(xd, f2(-1.0f), x);
                    k = fma2(muk, d, xd);
                    v = fma2(muv, d, xd);
                    r = fma2(mur, d, xd);
                } else {
                    const float2 xk = lds_pair<IO>(tK, o), xkd = lds_pair<IO>(tK + dsh, o);
                    const float2 xv = lds_pair<IO>(tV, o), xvd = lds_pair<IO>(tV + dsh, o);
                    k = fma2(muk, fma2(xkd, f2(-1.0f), xk), xkd);
                    v = fma2(muv, fma2(xvd, f2(-1.0f), xv), xvd);
                    if (GATE) {
                        const float2 xr = lds_pair<IO>(tR, o), xrd = lds_pair<IO>(tR + dsh, o);
                        r = fma2(mur, fma2(xrd, f2(-1.0f), xr), xrd);
                    }
                }
            } else {
                k = lds_pair<IO>(tK, o);
                v = lds_pair<IO>(tV, o);
                if (GATE) r = lds_pair<IO>(tR, o);
            }
            if (GATE) {
                float2 g = ex2(mul2(r, f2(-kLog2e)));
                // in k's slot the second half must follow the read of k, which
                // it does not depend on: tie it to k (no instruction)
                if (G1_IN_K) asm volatile("" : "+f"(g.y) : "f"(k.x), "f"(k.y));
                sts_f32(g0 + o, g.x);
                sts_f32(g1 + o, g.y);
            }
            kk[i] = k;
            vv[i] = v;
        }
        if (nv < kL) {
            // tokens past the sequence end: p = 0 and p v = 0
#pragma unroll
            for (int i = 0; i < kL; ++i) {
                kk[i] = (i < nv) ? kk[i] : f2(-INFINITY);
                vv[i] = (i < nv) ? vv[i] : f2(0.0f);
            }
        }
        float2 mx;
        mx.x = max3f(max3f(kk[0].x, kk[1].x, kk[2].x), max3f(kk[3].x, kk[4].x, kk[5].x), fmaxf(kk[6].x, kk[7].x));
        mx.y = max3f(max3f(kk[0].y, kk[1].y, kk[2].y), max3f(kk[3].y, kk[4].y, kk[5].y), fmaxf(kk[6].y, kk[7].y));
        Mh[st] = mx;
        const float2 negM = make_float2(mx.x == -INFINITY ? 0.0f : -mx.x * kLog2e,
                                        mx.y == -INFINITY ? 0.0f : -mx.y * kLog2e);
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            kk[i] = ex2(fma2(kk[i], f2(kLog2e), negM));  // p_i (0 beyond T)
            vv[i] = mul2(kk[i], vv[i]);                  // p_i v_i
        }
        // Two-sided sums inside the sub-chunk, both directions in one pass (four
        // independent recurrences per step): step it adds the forward sum
        // before token it and the backward sum after token 7 - it; a token's
        // second contribution also brings its own term e^u p v.
        float nd[32];  // per token i: num.x, num.y, den.x, den.y
        float2 fa = f2(0.0f), fc = f2(0.0f), ga = f2(0.0f), gc = f2(0.0f);
#pragma unroll
        for (int it = 0; it < kL; ++it) {
            const int i = it, ib = kL - 1 - it;
            if (it < kL / 2) {
                nd[4 * i + 0] = fa.x;
                nd[4 * i + 1] = fa.y;
                nd[4 * i + 2] = fc.x;
                nd[4 * i + 3] = fc.y;
                nd[4 * ib + 0] = ga.x;
                nd[4 * ib + 1] = ga.y;
                nd[4 * ib + 2] = gc.x;
                nd[4 * ib + 3] = gc.y;
            } else {
                const float2 n1 = add2(make_float2(nd[4 * i], nd[4 * i + 1]), fma2(eu, vv[i], fa));
                const float2 d1 = add2(make_float2(nd[4 * i + 2], nd[4 * i + 3]), fma2(eu, kk[i], fc));
                const float2 n2 = add2(make_float2(nd[4 * ib], nd[4 * ib + 1]), fma2(eu, vv[ib], ga));
                const float2 d2 = add2(make_float2(nd[4 * ib + 2], nd[4 * ib + 3]), fma2(eu, kk[ib], gc));
                nd[4 * i + 0] = n1.x;
                nd[4 * i + 1] = n1.y;
                nd[4 * i + 2] = d1.x;
                nd[4 * i + 3] = d1.y;
                nd[4 * ib + 0] = n2.x;
                nd[4 * ib + 1] = n2.y;
                nd[4 * ib + 2] = d2.x;
                nd[4 * ib + 3] = d2.y;
            }
            fa = fma2(alpha, fa, vv[i]);
            fc = fma2(alpha, fc, kk[i]);
            ga = fma2(alpha, ga, vv[ib]);
            gc = fma2(alpha, gc, kk[ib]);
        }
        // columns by step, not by sub-chunk: tcgen05.st takes one address for
        // the warp, and the output pass reads step st back at step st
        tmem_st32(tmem + st * 32, nd);
        Fh[st] = make_float4(fa.x, fa.y, fc.x, fc.y);
        Gh[st] = make_float4(ga.x, ga.y, gc.x, gc.y);
    }

    // ---- 3a. warp maximum (the reference of the warp's sums) and the chunk's
    // totals on it ---------------------------------------------------------------
    float2 mx = max2(max2(Mh[0], Mh[1]), max2(Mh[2], Mh[3]));
#pragma unroll
    for (int d = kNP; d < 32; d <<= 1) {
        mx.x = fmaxf(mx.x, __shfl_xor_sync(0xffffffffu, mx.x, d));
        mx.y = fmaxf(mx.y, __shfl_xor_sync(0xffffffffu, mx.y, d));
    }
    if (cq == 0) S.wmax[j][warp] = mx;  // -inf for a warp wholly past T
    const float2 mref = make_float2(mx.x == -INFINITY ? 0.0f : mx.x, mx.y == -INFINITY ? 0.0f : mx.y);
    float2 eh[kH];
    auto scale4 = [](float2 e, float4 v) {
        const float2 a = mul2(e, lo2(v)), c = mul2(e, hi2(v));
        return make_float4(a.x, a.y, c.x, c.y);
    };
#pragma unroll
    for (int st = 0; st < kH; ++st) {
        eh[st] = ex2(mul2(add2(Mh[st], make_float2(-mref.x, -mref.y)), f2(kLog2e)));
        Fh[st] = scale4(eh[st], Fh[st]);  // sub-chunk totals on the warp reference
        Gh[st] = scale4(eh[st], Gh[st]);
    }
    if (ROT) {
        // into natural sub-chunk order (each thread reads back its own entries)
#pragma unroll
        for (int st = 0; st < kH; ++st) {
            X2.a[(st + rot) & (kH - 1)][tid] = Fh[st];
            X2.b[(st + rot) & (kH - 1)][tid] = Gh[st];
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            Fh[h] = X2.a[h][tid];
            Gh[h] = X2.b[h][tid];
        }
    }
    // chunk totals: forward at the chunk's end, backward at its start
    float4 Fi = Fh[0], Gi = Gh[kH - 1];
#pragma unroll
    for (int h = 1; h < kH; ++h) {
        Fi = fma4(a8, Fi, Fh[h]);
        Gi = fma4(a8, Gi, Gh[kH - 1 - h]);
    }

    // ---- 3b. scans: warp, CTA, cluster ------------------------------------------
#pragma unroll
    for (int e = 0; (kNP << e) < 32; ++e) {
        // a^(32 * 2^e), zero where the partner lane lies outside the warp's chunks
        const float2 m = S.tab[1 << e][j];
        const float2 mf = cq >= (1 << e) ? m : f2(0.0f), mb = cq + (1 << e) < kCPW ? m : f2(0.0f);
        Fi = fma4(mf, shfl_up4(Fi, kNP << e, 32), Fi);
        Gi = fma4(mb, shfl_down4(Gi, kNP << e, 32), Gi);
    }
    float4 X = shfl_up4(Fi, kNP, 32), Y = shfl_down4(Gi, kNP, 32);
    if (cq == 0) X = zero4();
    if (cq == kCPW - 1) Y = zero4();
    if (cq == kCPW - 1) S.waggF[j][warp] = Fi;
    if (cq == 0) S.waggB[j][warp] = Gi;
    __syncthreads();
    // CTA scan, in every thread for its own pair (no warp waits on another's
    // serial scan): each warp's scale onto the CTA maximum, the folds of the
    // warps before and after this one, and the CTA's records for the column
    float4 XW = zero4(), YW = zero4();  // exclusive carries into this warp (CTA frame)
    float2 wsw = f2(0.0f);              // this warp's scale onto the CTA reference
    float4 ownF = zero4(), ownG = zero4();
    float2 ownM;
    {
        float2 mw[kNW];
        float4 sF[kNW], sB[kNW];
#pragma unroll
        for (int w = 0; w < kNW; ++w) mw[w] = S.wmax[j][w];
        const float2 mc = max2(max2(mw[0], mw[1]), max2(mw[2], mw[3]));
        const float2 a256 = S.tab[kCPW][j];  // across one warp's 256 tokens
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            // 2^(M_w - M_cta), 0 for a warp wholly past T
            const float2 sc = ex2(mul2(add2(mw[w], make_float2(-mc.x, -mc.y)), f2(kLog2e)));
            sF[w] = scale4(sc, S.waggF[j][w]);
            sB[w] = scale4(sc, S.waggB[j][w]);
            if (w == warp) wsw = sc;
        }
        // forward: the CTA's total sits at its last real warp (Tc may be
        // shorter than the CTA's capacity when the column spans several CTAs)
        const int wl = p.Tc / kWarpTok - 1;
        float4 acc = zero4();
#pragma unroll
        for (int w = 0; w < kNW; ++w) {
            if (w == warp) XW = acc;
            acc = fma4(a256, acc, sF[w]);
            if (w == wl) ownF = acc;
        }
        acc = zero4();
#pragma unroll
        for (int w = kNW - 1; w >= 0; --w) {
            if (w == warp) YW = acc;
            acc = fma4(a256, acc, sB[w]);
        }
        ownG = acc;
        ownM = mul2(mc, f2(kLog2e));  // base 2, the unit of the exponents below
    }
    // column exchange: every CTA's records reach every CTA of the column;
    // each thread then folds them for its pair
    float2 cs_sl = f2(1.0f), cs_af = f2(0.0f), cs_cf = f2(0.0f), cs_bb = f2(0.0f), cs_db = f2(0.0f);
    if (p.ncl > 1) {
        if (GX) {
            // publish the record to the workspace, then the flag (release
            // after every writer's fence), then wait for the column's flags
            // and copy the records into the mailbox
            if (q == 0) {
                S.ownF[j] = ownF;
                S.ownG[j] = ownG;
                S.ownM[j] = ownM;
            }
            __syncthreads();
            float4* rec = p.ws_rec + ((size_t)col * fast::kClusterMax + rank) * fast::kRecF4;
            if (tid < fast::kRecF4) {
                float4 v;
                if (tid < kNP) {
                    v = S.ownF[tid];
                } else if (tid < 2 * kNP) {
                    v = S.ownG[tid - kNP];
                } else {
                    const int m = 2 * (tid - 2 * kNP);
                    v = make_float4(S.ownM[m].x, S.ownM[m].y, S.ownM[m + 1].x, S.ownM[m + 1].y);
                }
                __stcg(rec + tid, v);
                __threadfence();
            }
            __syncthreads();
            unsigned int* flags = p.ws_flag + (size_t)col * fast::kClusterMax;
            if (tid == 0)
                asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flags + rank), "r"(gen + 1u) : "memory");
            if (tid < p.ncl) fast::wait_flag(flags + tid, gen + 1u, p.err);
            __syncthreads();
            const float4* peers = p.ws_rec + (size_t)col * fast::kClusterMax * fast::kRecF4;
            for (int e = tid; e < p.ncl * fast::kRecF4; e += kThreads) {
                const int r = e / fast::kRecF4, k = e - r * fast::kRecF4;
                const float4 v = __ldcg(peers + e);
                if (k < kNP) {
                    S.mbF[r][k] = v;
                } else if (k < 2 * kNP) {
                    S.mbG[r][k - kNP] = v;
                } else {
                    const int m = 2 * (k - 2 * kNP);
                    S.mbM[r][m] = make_float2(v.x, v.y);
                    S.mbM[r][m + 1] = make_float2(v.z, v.w);
                }
            }
            __syncthreads();
        } else {
            // asynchronous stores into every CTA's mailbox (its own included):
            // thread (pair j, chunk q) sends pair j's forward record to peer q
            // (q < ncl), its backward record and maximum to peer q - ncl
            // (ncl <= q < 2 ncl); each thread then waits, bounded, until its
            // CTA's mailbox is full
            cluster_wait_acquire();  // every mailbox barrier is initialised
            if (q < 2 * p.ncl) {
                const int peer = q < p.ncl ? q : q - p.ncl;
                const unsigned rbar = mapa_u32(smem_u32(&S.xbar), peer);
                if (q < p.ncl) {
                    st_async4(mapa_u32(smem_u32(&S.mbF[rank][j]), peer), ownF, rbar);
                } else {
                    st_async4(mapa_u32(smem_u32(&S.mbG[rank][j]), peer), ownG, rbar);
                    st_async2(mapa_u32(smem_u32(&S.mbM[rank][j]), peer), ownM, rbar);
                }
            }
            mbar_wait_cluster_bounded(&S.xbar, p.err);
        }
        // fold the peers' records on the column maximum: the forward ones of
        // the CTAs before this one, the backward ones of those after it, each
        // CTA a decay of a^Tc further
        const float2 aTc = ex2c(mul2(lam2, f2(-(float)p.Tc)));
        // (loops of exactly the peers' count: rank and ncl are the same in
        // every thread of the CTA)
        float2 Mc = f2(-INFINITY);
#pragma unroll 1
        for (int r = 0; r < p.ncl; ++r) Mc = max2(Mc, S.mbM[r][j]);
        float4 accF = zero4(), accG = zero4();
#pragma unroll 1
        for (int r = 0; r < rank; ++r) {
            const float2 sc = ex2(add2(S.mbM[r][j], make_float2(-Mc.x, -Mc.y)));
            accF = fma4(aTc, accF, scale4(sc, S.mbF[r][j]));
        }
#pragma unroll 1
        for (int r = p.ncl - 1; r > rank; --r) {
            const float2 sc = ex2(add2(S.mbM[r][j], make_float2(-Mc.x, -Mc.y)));
            accG = fma4(aTc, accG, scale4(sc, S.mbG[r][j]));
        }
        cs_sl = ex2(add2(ownM, make_float2(-Mc.x, -Mc.y)));
        cs_af = lo2(accF);
        cs_cf = hi2(accF);
        cs_bb = lo2(accG);
        cs_db = hi2(accG);
    }

    // ---- 4. carries -> outputs ---------------------------------------------------
    const float2 sl = cs_sl;
    const float2 slw = mul2(sl, wsw);
    const float2 slF = mul2(sl, S.tab[cq][j]), slB = mul2(sl, S.tab[kCPW - 1 - cq][j]);
    const float2 kf = S.tab[q][j];                          // CTA start -> chunk start
    const float2 kb = S.tab[max(0, p.Tc / kKL - 1 - q)][j];  // chunk end -> CTA end
    // carries into the chunk: from the left at its start, from the right at its end
    float2 Ac = fma2(slw, lo2(X), fma2(slF, lo2(XW), mul2(kf, cs_af)));
    float2 Cc = fma2(slw, hi2(X), fma2(slF, hi2(XW), mul2(kf, cs_cf)));
    // carries into each sub-chunk, natural order: from the right, B_3 = the
    // chunk's and B_{h-1} = a^8 B_h + G_h; from the left, A_0 = the chunk's
    // and A_{h+1} = a^8 A_h + F_h (sub-chunk totals on the column reference)
    float4 Lc[kH], Rc[kH];  // (A.xy, C.xy), (B.xy, D.xy)
    {
        float2 Bq = fma2(slw, lo2(Y), fma2(slB, lo2(YW), mul2(kb, cs_bb)));
        float2 Dq = fma2(slw, hi2(Y), fma2(slB, hi2(YW), mul2(kb, cs_db)));
#pragma unroll
        for (int h = kH - 1; h >= 0; --h) {
            Rc[h] = make_float4(Bq.x, Bq.y, Dq.x, Dq.y);
            if (h > 0) {
                Bq = fma2(slw, lo2(Gh[h]), mul2(a8, Bq));
                Dq = fma2(slw, hi2(Gh[h]), mul2(a8, Dq));
            }
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            Lc[h] = make_float4(Ac.x, Ac.y, Cc.x, Cc.y);
            Ac = fma2(slw, lo2(Fh[h]), mul2(a8, Ac));
            Cc = fma2(slw, hi2(Fh[h]), mul2(a8, Cc));
        }
    }
    if (ROT) {
#pragma unroll
        for (int h = 0; h < kH; ++h) {
            X2.a[h][tid] = Lc[h];
            X2.b[h][tid] = Rc[h];
        }
    }
    float2 pw[kL];
    pw[0] = f2(1.0f);
#pragma unroll
    for (int i = 1; i < kL; ++i) pw[i] = min2(mul2(pw[i - 1], alpha), f2(0x1p126f));
    tmem_wait_st();
    char* tout = smem;
#pragma unroll
    for (int st = 0; st < kH; ++st) {
        const int h = ROT ? (st + rot) & (kH - 1) : st;
        float nd[32];
        tmem_ld32(tmem + st * 32, nd);  // the sums of sub-chunk h, stored at this step
        const float2 sh = mul2(slw, eh[st]);
        const float4 L4 = ROT ? X2.a[h][tid] : Lc[st], R4 = ROT ? X2.b[h][tid] : Rc[st];
        const float2 Ah = lo2(L4), Ch = hi2(L4), Bh = lo2(R4), Dh = hi2(R4);
        const int rowoff = (q * kH + h) * RB + j * PB;
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            const int o = rowoff + i * SUB;
            const float2 nn = make_float2(nd[4 * i], nd[4 * i + 1]);
            const float2 dd = make_float2(nd[4 * i + 2], nd[4 * i + 3]);
            const float2 num = fma2(sh, nn, fma2(pw[i], Ah, mul2(pw[kL - 1 - i], Bh)));
            float2 den = fma2(sh, dd, fma2(pw[i], Ch, mul2(pw[kL - 1 - i], Dh)));
            if (GATE) {
                // read before the result overwrites the first slot
                const float2 g = make_float2(lds_f32(g0 + o), lds_f32(g1 + o));
                den = fma2(den, g, den);
            }
            Io<IO>::st_pair(tout + o, mul2(num, rcp(den)));
        }
    }
    // results leave by TMA stores: lane i of warp 0 stores sub-tile i in boxes
    // of 256 strided tokens, clipped at T by the tensor map
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < kL) {
        if (p.ofold) {
            if (tid == 0) fast::tma_store_4d(&p.omap, tout, c0, t0 / kL, 0, b);
        } else {
            const int nbox = (tend - t0 + 255) / 256;
            for (int hb = 0; hb < nbox; ++hb)
                tma_store_3d(&p.omap, tout + tid * SUB + hb * 32 * RB, c0, t0 + tid + 256 * hb, b);
        }
        bulk_commit_and_wait_read();
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(S.tmem), "r"(kTmemCols)
                     : "memory");
    }
    if (GX && tid == 0) {
        // count the CTA out; the last one resets the counters for the next
        // launch and advances the generation
        __threadfence();
        const unsigned int d = atomicAdd(p.ws_ctl + 1, 1u);
        if (d == (unsigned int)p.total - 1u) {
            atomicExch(p.ws_ctl + 0, 0u);
            atomicExch(p.ws_ctl + 1, 0u);
            __threadfence();
            atomicExch(p.ws_ctl + 2, gen + 1u);
        }
    }
}

}  // namespace tm32
}  // namespace vrwkv
