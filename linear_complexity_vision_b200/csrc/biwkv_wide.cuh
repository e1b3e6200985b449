// Fused Q-Shift -> Bi-WKV -> sigma(R) gate on 16-channel slabs, sm_100a.
//
// Evaluates Bi-WKV of "Vision-RWKV Backbone", Linear Complexity
// Bidirectional Attention, eq. 5, on inputs Q-Shifted per Quad-Directional
// Token Shift, eq. 9, gated per Overall Architecture, eq. 2, as a chunked
// two-sided linear scan:
//
//   A_t = sum_{i<t} a^{t-1-i} p_i v_i,  B_t = sum_{i>t} a^{i-t-1} p_i v_i,
//   C_t, D_t with v = 1,  a = e^{-w/T},  p_i = e^{k_i - M},
//   wkv_t = (A_t + B_t + e^u p_t v_t) / (C_t + D_t + e^u p_t).
//
// Work decomposition.  A CTA owns batch row b, a slab of 16 channels and
// 512 tokens; its 256 threads are 8 channel pairs x 32 chunks of 16 tokens
// (lane = pair + 8 * (chunk mod 4), warp = chunk / 4).  Longer sequences
// split over a thread-block cluster of up to 8 CTAs along T.
//
//  1. Tiles arrive by TMA (cp.async.bulk.tensor, no multicast) from a 4-D
//     view (C, 16, T/16, B) of each (B, T, C) input with a box of 17 token
//     rows per 16-token chunk: the 17th row lies outside the view and is
//     zero-filled, so chunks sit 17 rows apart in shared memory and the four
//     chunks a warp reads at once fall in different banks.  Q-Shift's
//     neighbour comes from the same tile: the vertical groups read the row
//     s*W tokens away (halo chunks loaded with the tile; chunks outside the
//     image are zero-filled, which is Q-Shift's zero border), the horizontal
//     groups (shift 1) take the previous or next token's value, which the
//     thread loaded one step earlier or later, with the chunk's first or
//     last neighbour read from the adjacent chunk unless it lies across the
//     row's end (W is a multiple of 16, so rows start on chunk boundaries).
//  2. Each thread mixes its 16 tokens (k, v, r), parks e^{-r} in shared
//     memory and keeps k and v in registers; the CTA's maximum of k per
//     channel becomes the exponent reference of every p in the CTA, so no
//     per-token rescaling is needed later.
//  3. p = 2^{(k - M) log2 e}, p v; Horner sums give each 8-token
//     sub-chunk's forward and backward totals.
//  4. The 32 chunk totals of a channel pair are scanned by one warp with its
//     lanes as chunks (warp j holds pair j): five shuffle levels.  Across
//     the cluster, every CTA pushes its totals and maximum into each peer's
//     shared-memory mailbox with asynchronous stores completing on the
//     peer's mbarrier; lanes then take the role of peers, rescale to the
//     column maximum and scan once more; the column carry comes back into
//     the CTA's exponent frame by one factor (exponent capped at 64, enough
//     for |w|, |u| and the k spread the limits allow).
//     Sequences longer than 8 CTAs (4096 tokens) split into segments of one
//     cluster each (SEG kernels, which need a caller-provided workspace):
//     clusters take tickets from a counter in the workspace, so the segments
//     of a column start in order; after its own exchange, each segment
//     publishes its totals and maximum (a record and a flag tagged with the
//     launch's generation) and every CTA waits, bounded, for the other
//     segments of its column, rescales their records to the column maximum,
//     scans them and adds the carries from earlier and later segments.
//  5. Per 8-token sub-chunk: a forward walk from the carry keeps
//     A_t + e^u p_t v_t (and the denominator) in registers, a backward walk
//     adds B_t and writes num / (den (1 + e^{-r})) into the tile, which then
//     leaves by coalesced 16-byte stores.
// Exponents are base 2 (log2 e is folded into k, u, w and r).
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "biwkv_tma.cuh"

namespace vrwkv {
namespace wide {

constexpr int kCW = 16;          // channels per CTA
constexpr int kNP = kCW / 2;     // channel pairs per CTA (= warps per CTA)
constexpr int kL = 16;           // tokens per thread chunk
constexpr int kS = 8;            // tokens per sub-chunk of the output walks
constexpr int kThreads = 256;    // kNP pairs x 32 chunks
constexpr int kChunks = 32;      // chunks per CTA
constexpr int kTc = kChunks * kL;  // tokens per CTA
constexpr int kRows = kL + 1;    // shared-memory rows per chunk (one zero pad row)
constexpr int kBoxChunks = 4;    // chunks per TMA box
constexpr int kClusterMax = 8;
constexpr int kHaloMax = 16;     // halo chunks on one side (s*W <= 256 tokens)
constexpr float kCarryExpCap = 64.0f;  // cap of the exponent lifting a column carry into the CTA frame

enum Layout { kKV = 0, kRKV = 1, kX = 2 };

// Q-Shift mode of a CTA's channels (uniform per CTA: every group bound is a
// multiple of 16): the source of x_shift.
enum Mode { kFromLeft = 0, kFromRight = 1, kFromUp = 2, kFromDown = 3, kSelf = 4 };

struct alignas(64) Params {
    CUtensorMap map[3];  // 4-D views (C, 16, T/16, B) of the distinct sources
    const float* w;
    const float* u;
    const float* mu[3];  // mu of r, k, v (each nullable)
    char* out;
    unsigned int* err;
    int B, T, C;
    int W, s;            // Q-Shift grid width and shift
    QsBounds g;          // Q-Shift channel-group bounds (multiples of 16)
    int ng;              // shifted groups: 4 (Q-Shift) or 2 (bidirectional shift)
    int qs;              // Q-Shift on (else the inputs are used as they are)
    float invT;          // 1 / T
    int nchunkT;         // T / 16
    int ncl;             // CTAs per cluster (a column, or one segment of it)
    int hv;              // vertical halo in chunks: s * W / 16 (<= kHaloMax)
    // segmented columns (SEG kernels only)
    int nseg;            // clusters (segments of ncl * 512 tokens) per column
    int nslab;           // channel slabs: C / 16
    int total;           // CTAs in the grid
    unsigned int* ws_ctl;   // [0] ticket counter, [1] finished CTAs, [2] generation
    unsigned int* ws_flag;  // per (column, segment): generation + 1 once its record is out
    float4* ws_rec;         // per (column, segment, pair): F, G, (M, 0, 0)
};

// Record one CTA sends to every peer of its column: per pair, the forward
// total (A.xy, C.xy), the backward total (B.xy, D.xy) and the maximum of k
// (base 2).
struct alignas(16) Rec {
    float4 F, G;
    float2 M;
    float2 pad;
};

struct alignas(16) Scratch {
    float2 pw16[kChunks][kNP];   // a^(16 l), l = 0..31, per pair
    float2 alpha[kNP], a8[kNP], eu[kNP];
    float2 acl[3][kNP];          // a^(512 d), d = 1, 2, 4: across CTAs
    float2 aseg[3][kNP];         // a^(512 ncl d), d = 1, 2, 4: across segments (SEG)
    int tk;                      // SEG: this cluster's ticket
    unsigned int gen;            // SEG: the launch's generation
    int mkey[kCW];               // CTA maximum of k per channel (ordered-int encoding)
    // chunk forward / backward totals, then the carries into each chunk; one
    // float4 of row padding: the scan warps read down a column (32 chunks of
    // one pair), which without it would hit the same four banks
    float4 aggF[kChunks][kNP + 1];
    float4 aggG[kChunks][kNP + 1];
    Rec own[kNP];                // this CTA's record
    Rec mb[kClusterMax][kNP];    // mailbox: every peer's record (own included)
    unsigned long long bar;      // TMA completion barrier
    unsigned long long xbar;     // mailbox barrier
};

// Monotone int encoding of floats for atomicMax (-inf < every finite < +inf).
__device__ __forceinline__ int fkey(float f) {
    const int i = __float_as_int(f);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float fkey_inv(int k) { return __int_as_float(k >= 0 ? k : k ^ 0x7fffffff); }

template <typename IO>
__device__ __forceinline__ unsigned lds_word(const char* p);
template <>
__device__ __forceinline__ unsigned lds_word<__nv_bfloat16>(const char* p) {
    return *reinterpret_cast<const unsigned*>(p);
}
// bf16 pair word -> float2 (integer unpack)
__device__ __forceinline__ float2 unpack_bf16(unsigned u) {
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// Channel pair of one token from a tile.
template <typename IO>
__device__ __forceinline__ float2 ld2(const char* p);
template <>
__device__ __forceinline__ float2 ld2<__nv_bfloat16>(const char* p) {
    return unpack_bf16(*reinterpret_cast<const unsigned*>(p));
}
template <>
__device__ __forceinline__ float2 ld2<float>(const char* p) {
    return *reinterpret_cast<const float2*>(p);
}

template <typename IO>
__device__ __forceinline__ void st2(char* p, float2 v);
template <>
__device__ __forceinline__ void st2<__nv_bfloat16>(char* p, float2 v) {
    *reinterpret_cast<__nv_bfloat162*>(p) = __float22bfloat162_rn(v);
}
template <>
__device__ __forceinline__ void st2<float>(char* p, float2 v) {
    *reinterpret_cast<float2*>(p) = v;
}

__device__ __forceinline__ float4 f4(float2 a, float2 b) { return make_float4(a.x, a.y, b.x, b.y); }
// three-input maximum (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float4 fma4(float2 m, float4 x, float4 y) {
    return f4(fma2(m, fast::lo2(x), fast::lo2(y)), fma2(m, fast::hi2(x), fast::hi2(y)));
}
__device__ __forceinline__ float4 scale4(float2 m, float4 x) {
    return f4(mul2(m, fast::lo2(x)), mul2(m, fast::hi2(x)));
}
__device__ __forceinline__ float4 shfl_idx4(float4 v, int src) {
    return make_float4(__shfl_sync(0xffffffffu, v.x, src), __shfl_sync(0xffffffffu, v.y, src),
                       __shfl_sync(0xffffffffu, v.z, src), __shfl_sync(0xffffffffu, v.w, src));
}

// Phase 1 for one thread's chunk: load, Q-Shift mix, gate factor (parked),
// k and v kept.  MODE is the CTA's Q-Shift mode; NSRC the distinct sources.
template <typename IO, int LAYOUT, bool QS, int MODE>
__device__ __forceinline__ void load_chunk(const char* const* tb, int hoff, bool left_ok, bool right_ok,
                                           float2 muk, float2 muv, float2 mur, float2* park, int park_stride,
                                           float2 (&kk)[kL], float2 (&vv)[kL]) {
    constexpr int es = Io<IO>::kBytes;
    constexpr int RB = kCW * es;  // bytes per token row
    constexpr int CB = kRows * RB;
    constexpr bool GATE = LAYOUT != kKV;
    constexpr int NSRC = LAYOUT == kKV ? 2 : (LAYOUT == kRKV ? 3 : 1);
    // source order in tb: kX {x}; kKV {k, v}; kRKV {r, k, v}
    constexpr int SK = LAYOUT == kRKV ? 1 : 0;
    constexpr int SV = LAYOUT == kKV ? 1 : (LAYOUT == kRKV ? 2 : 0);
    constexpr int SR = 0;
    float2 cur[NSRC], nxt[NSRC], prv[NSRC];
#pragma unroll
    for (int s = 0; s < NSRC; ++s) {
        cur[s] = ld2<IO>(tb[s]);
        if (QS && MODE == kFromLeft) prv[s] = left_ok ? ld2<IO>(tb[s] - CB + (kL - 1) * RB) : f2(0.0f);
    }
#pragma unroll
    for (int i = 0; i < kL; ++i) {
        float2 xd[NSRC];
#pragma unroll
        for (int s = 0; s < NSRC; ++s) {
            if (QS && MODE == kFromRight) {
                if (i + 1 < kL) nxt[s] = ld2<IO>(tb[s] + (i + 1) * RB);
                else nxt[s] = right_ok ? ld2<IO>(tb[s] + CB) : f2(0.0f);
                xd[s] = nxt[s];
            } else if (QS && MODE == kFromLeft) {
                xd[s] = prv[s];
            } else if (QS && (MODE == kFromUp || MODE == kFromDown)) {
                xd[s] = ld2<IO>(tb[s] + i * RB + hoff);
            } else {
                xd[s] = cur[s];
            }
        }
        float2 k, v, r;
        if (QS && MODE != kSelf) {
            if (LAYOUT == kX) {
                const float2 d = add2(cur[0], make_float2(-xd[0].x, -xd[0].y));
                k = fma2(muk, d, xd[0]);
                v = fma2(muv, d, xd[0]);
                r = fma2(mur, d, xd[0]);
            } else {
                k = fma2(muk, add2(cur[SK], make_float2(-xd[SK].x, -xd[SK].y)), xd[SK]);
                v = fma2(muv, add2(cur[SV], make_float2(-xd[SV].x, -xd[SV].y)), xd[SV]);
                if (GATE) r = fma2(mur, add2(cur[SR], make_float2(-xd[SR].x, -xd[SR].y)), xd[SR]);
            }
        } else {
            k = cur[SK];
            v = cur[SV];
            r = cur[SR];
        }
        if (GATE) park[i * park_stride] = ex2(mul2(r, f2(-kLog2e)));
        kk[i] = k;
        vv[i] = v;
        // advance the sliding neighbours
#pragma unroll
        for (int s = 0; s < NSRC; ++s) {
            if (QS && MODE == kFromLeft) prv[s] = cur[s];
            if (i + 1 < kL) {
                if (QS && MODE == kFromRight) cur[s] = nxt[s];
                else cur[s] = ld2<IO>(tb[s] + (i + 1) * RB);
            }
        }
    }
}

// Bounded wait for a flag (acquire); records bit 1 of the error word.
__device__ __forceinline__ void wait_flag_bounded(const unsigned int* f, unsigned int want, unsigned int* err) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v == want) return;
    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
    for (;;) {
        __nanosleep(64);
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v == want) return;
        if (fast::global_ns() - t0 > lim) {
            atomicOr(err, 2u);
            return;
        }
    }
}

template <typename IO, int LAYOUT, bool QS, bool SEG>
__global__ void __launch_bounds__(kThreads, 2) biwkv_wide_kernel(const __grid_constant__ Params p) {
    constexpr int es = Io<IO>::kBytes;
    constexpr int RB = kCW * es;
    constexpr int CB = kRows * RB;
    constexpr int PB = 2 * es;
    constexpr bool GATE = LAYOUT != kKV;
    constexpr int NSRC = LAYOUT == kKV ? 2 : (LAYOUT == kRKV ? 3 : 1);

    extern __shared__ __align__(128) char smem_raw[];
    char* smem = smem_raw + ((128u - (fast::smem_u32(smem_raw) & 127u)) & 127u);
    Scratch& S = *reinterpret_cast<Scratch*>(smem);

    const int tid = threadIdx.x;
    const int j = tid & (kNP - 1);          // channel pair
    const int warp = tid >> 5;
    const int q = warp * 4 + ((tid >> 3) & 3);  // chunk within the CTA
    const int rank = blockIdx.x;  // rank in the cluster
    int slab = blockIdx.y, b = blockIdx.z, seg = 0, col = 0;
    unsigned int gen = 0;
    if (SEG) {
        // the cluster's rank 0 takes a ticket and hands it to every CTA of the
        // cluster: segments of a column hold consecutive tickets.  The first
        // cluster barrier makes sure every CTA runs before its shared memory
        // is written, the second publishes the ticket.
        fast::cluster_arrive_relaxed();
        fast::cluster_wait_acquire();
        if (rank == 0 && tid == 0) {
            const int t = (int)atomicAdd(p.ws_ctl, 1u);
            const unsigned int g = *reinterpret_cast<volatile unsigned int*>(p.ws_ctl + 2);
            for (int r = 0; r < p.ncl; ++r) {
                asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(fast::mapa_u32(fast::smem_u32(&S.tk), r)),
                             "r"(t)
                             : "memory");
                asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(fast::mapa_u32(fast::smem_u32(&S.gen), r)),
                             "r"(g)
                             : "memory");
            }
        }
        fast::cluster_arrive_release();
        fast::cluster_wait_acquire();
        const int t = S.tk;
        if (t < 0 || t >= p.total / p.ncl) {  // a workspace that was not zero-filled
            if (tid == 0) atomicOr(p.err, 4u);
            return;
        }
        gen = S.gen;
        col = t / p.nseg;
        seg = t - col * p.nseg;
        slab = col % p.nslab;
        b = col / p.nslab;
    }
    const int grank = seg * p.ncl + rank;  // CTA index along the column
    const int c0 = slab * kCW;
    const int t0 = grank * kTc;

    // Q-Shift mode of this slab and the tile's halo (chunks before / after)
    int mode = kSelf;
    if (QS && p.s > 0) {
        int grp = qs_group(c0, p.g);
        if (grp >= p.ng) grp = 4;
        mode = grp;  // kFromLeft .. kFromDown, kSelf
    }
    int hb = 0, ha = 0;
    if (mode == kFromLeft) hb = 1;
    if (mode == kFromRight) ha = 1;
    if (mode == kFromUp) hb = p.hv;
    if (mode == kFromDown) ha = p.hv;
    const int hb4 = (hb + kBoxChunks - 1) / kBoxChunks * kBoxChunks;
    const int ha4 = (ha + kBoxChunks - 1) / kBoxChunks * kBoxChunks;
    const int tchunks = kChunks + hb4 + ha4;
    const int tile_bytes = tchunks * CB;
    char* tiles = smem + ((sizeof(Scratch) + 127) & ~size_t(127));
    float2* park = reinterpret_cast<float2*>(tiles + NSRC * tile_bytes);  // [token in chunk][chunk][pair]

    if (tid == 0) {
        fast::mbar_init(&S.bar, 1);
        if (p.ncl > 1) {
            fast::mbar_init(&S.xbar, 1);
            fast::mbar_expect_tx(&S.xbar, (unsigned)(p.ncl * kNP * sizeof(Rec)));
        }
    }
    if (tid < kCW) S.mkey[tid] = fkey(-INFINITY);
    // decay and bonus tables: a^(16 l) per pair (one entry per thread), and
    // a, a^8, e^u, a^(512 d) per pair
    const float lam_scale = p.invT * kLog2e;
    {
        const int l = tid >> 3, jj = tid & 7;
        const float2 lam = mul2(make_float2(__ldg(p.w + c0 + 2 * jj), __ldg(p.w + c0 + 2 * jj + 1)),
                                f2(lam_scale));
        S.pw16[l][jj] = ex2c(mul2(lam, f2(-16.0f * l)));
        if (l == 0) {
            S.alpha[jj] = ex2c(make_float2(-lam.x, -lam.y));
            S.a8[jj] = ex2c(mul2(lam, f2(-8.0f)));
        } else if (l == 1) {
            S.eu[jj] = ex2(mul2(make_float2(__ldg(p.u + c0 + 2 * jj), __ldg(p.u + c0 + 2 * jj + 1)),
                                f2(kLog2e)));
        } else if (l >= 2 && l < 5) {
            S.acl[l - 2][jj] = ex2c(mul2(lam, f2(-(float)kTc * (float)(1 << (l - 2)))));
        } else if (SEG && l >= 5 && l < 8) {
            S.aseg[l - 5][jj] = ex2c(mul2(lam, f2(-(float)kTc * (float)p.ncl * (float)(1 << (l - 5)))));
        }
    }
    __syncthreads();
    if (p.ncl > 1) fast::cluster_arrive_relaxed();

    // ---- tile loads: lane i of warp 0 loads box i of each source ---------
    const int nbox = tchunks / kBoxChunks;
    if (warp == 0) {
        if (tid == 0) fast::mbar_expect_tx(&S.bar, (unsigned)(NSRC * nbox * kBoxChunks * CB));
        __syncwarp();
        const int qlo = grank * kChunks - hb4;
        for (int i = tid; i < NSRC * nbox; i += 32) {
            const int s = i / nbox, bx = i - s * nbox;
            char* dst = tiles + s * tile_bytes + bx * kBoxChunks * CB;
            fast::tma_load_4d(dst, &p.map[s], c0, 0, qlo + bx * kBoxChunks, b, &S.bar);
        }
    }

    // ---- per-thread constants (overlap the copies) ------------------------
    const int cA = c0 + 2 * j;
    auto mu_of = [&](const float* m) {
        return m ? make_float2(__ldg(m + cA), __ldg(m + cA + 1)) : f2(0.0f);
    };
    const float2 muk = QS ? mu_of(p.mu[1]) : f2(1.0f);
    const float2 muv = QS ? mu_of(p.mu[2]) : f2(1.0f);
    const float2 mur = (QS && GATE) ? mu_of(p.mu[0]) : f2(1.0f);
    const int qg = grank * kChunks + q;          // chunk within the column
    const bool valid = qg < p.nchunkT;           // chunks past T hold no tokens
    const int wstart = (qg * kL) % max(p.W, 1);  // column of the chunk's first token
    const bool left_ok = wstart > 0;             // the token before the chunk is in its row
    const bool right_ok = wstart + kL < p.W;     // the token after the chunk is in its row
    const int hoff = (mode == kFromUp ? -p.hv : p.hv) * CB;

    if (tid == 0) fast::mbar_wait_bounded(&S.bar, p.err);
    __syncthreads();

    // ---- 1-2. load, mix, park e^{-r}; k and v to registers -----------------
    const char* tb[NSRC];
#pragma unroll
    for (int s = 0; s < NSRC; ++s) tb[s] = tiles + s * tile_bytes + (q + hb4) * CB + j * PB;
    float2* mypark = park + q * kNP + j;
    constexpr int park_stride = kChunks * kNP;
    float2 kk[kL], vv[kL];
    switch (mode) {
    case kFromLeft:
        load_chunk<IO, LAYOUT, QS, kFromLeft>(tb, hoff, left_ok, right_ok, muk, muv, mur, mypark, park_stride, kk, vv);
        break;
    case kFromRight:
        load_chunk<IO, LAYOUT, QS, kFromRight>(tb, hoff, left_ok, right_ok, muk, muv, mur, mypark, park_stride, kk, vv);
        break;
    case kFromUp:
    case kFromDown:
        load_chunk<IO, LAYOUT, QS, kFromUp>(tb, hoff, left_ok, right_ok, muk, muv, mur, mypark, park_stride, kk, vv);
        break;
    default:
        load_chunk<IO, LAYOUT, QS, kSelf>(tb, hoff, left_ok, right_ok, muk, muv, mur, mypark, park_stride, kk, vv);
        break;
    }
    // CTA maximum of k per channel: warp lanes of one pair, then one atomic.
    // A chunk past T (zero-filled by the TMA) takes no part in the maximum,
    // and its p and p v are zeroed below.
    float2 mx = f2(-INFINITY);
#pragma unroll
    for (int i = 0; i < kL; i += 2) {
        mx.x = fmax3(mx.x, kk[i].x, kk[i + 1].x);
        mx.y = fmax3(mx.y, kk[i].y, kk[i + 1].y);
    }
    if (!valid) mx = f2(-INFINITY);
#pragma unroll
    for (int d = 8; d < 32; d <<= 1) {
        mx.x = fmaxf(mx.x, __shfl_xor_sync(0xffffffffu, mx.x, d));
        mx.y = fmaxf(mx.y, __shfl_xor_sync(0xffffffffu, mx.y, d));
    }
    if ((tid & 31) < kNP) {
        atomicMax(&S.mkey[2 * j], fkey(mx.x));
        atomicMax(&S.mkey[2 * j + 1], fkey(mx.y));
    }
    __syncthreads();

    // ---- 3. p, p v (in place) and sub-chunk totals --------------------------
    const float2 Mcta = make_float2(fkey_inv(S.mkey[2 * j]), fkey_inv(S.mkey[2 * j + 1]));
    // a CTA whose tokens all lie past T has M = -inf: reference 0 (p = 0 there)
    // a chunk past T gets p = 2^-inf = 0 (its k are the zero fill)
    const float2 negM = !valid ? f2(-INFINITY)
                               : make_float2(Mcta.x == -INFINITY ? 0.0f : -Mcta.x * kLog2e,
                                             Mcta.y == -INFINITY ? 0.0f : -Mcta.y * kLog2e);
    const float2 alpha = S.alpha[j], a8 = S.a8[j];
    float4 Fs[2], Gs[2];  // per sub-chunk: forward and backward totals (num.xy, den.xy)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float2 fa = f2(0.0f), fc = f2(0.0f), ga = f2(0.0f), gc = f2(0.0f);
#pragma unroll
        for (int i = 0; i < kS; ++i) {
            const int t = h * kS + i;
            kk[t] = ex2(fma2(kk[t], f2(kLog2e), negM));  // p
            vv[t] = mul2(kk[t], vv[t]);                  // p v
            fa = fma2(alpha, fa, vv[t]);
            fc = fma2(alpha, fc, kk[t]);
        }
#pragma unroll
        for (int i = kS - 1; i >= 0; --i) {
            const int t = h * kS + i;
            ga = fma2(alpha, ga, vv[t]);
            gc = fma2(alpha, gc, kk[t]);
        }
        Fs[h] = f4(fa, fc);
        Gs[h] = f4(ga, gc);
    }
    // chunk totals: forward referenced to the chunk's last token, backward to
    // its first
    S.aggF[q][j] = fma4(a8, Fs[0], Fs[1]);
    S.aggG[q][j] = fma4(a8, Gs[1], Gs[0]);
    __syncthreads();

    // ---- 4. scans: warp `warp` holds pair `warp`, lane l = chunk l ----------
    {
        const int jj = warp, l = tid & 31;
        float4 F = S.aggF[l][jj], G = S.aggG[l][jj];
#pragma unroll
        for (int e = 0; e < 5; ++e) {
            const int d = 1 << e;
            const float2 m = S.pw16[d][jj];  // a^(16 d)
            const float4 uF = fast::shfl_up4(F, d, 32);
            const float4 dG = fast::shfl_down4(G, d, 32);
            if (l >= d) F = fma4(m, uF, F);
            if (l + d < 32) G = fma4(m, dG, G);
        }
        // exclusive carries into chunk l (zero at the CTA's ends)
        float4 cF = fast::shfl_up4(F, 1, 32), cG = fast::shfl_down4(G, 1, 32);
        if (l == 0) cF = fast::zero4();
        if (l == 31) cG = fast::zero4();
        const float4 Fcta = shfl_idx4(F, 31), Gcta = shfl_idx4(G, 0);
        if (p.ncl > 1) {
            if (l == 0) {
                const float2 mb2 = make_float2(fkey_inv(S.mkey[2 * jj]), fkey_inv(S.mkey[2 * jj + 1]));
                S.own[jj].F = Fcta;
                S.own[jj].G = Gcta;
                S.own[jj].M = mul2(mb2, f2(kLog2e));
            }
            __syncwarp();
            // push the record to every peer (own mailbox included), lane l -> peer l
            fast::cluster_wait_acquire();
            if (l < p.ncl) {
                const unsigned rbar = fast::mapa_u32(fast::smem_u32(&S.xbar), l);
                const unsigned dst = fast::mapa_u32(fast::smem_u32(&S.mb[rank][jj]), l);
                const Rec& r = S.own[jj];
                fast::st_async4(dst, r.F, rbar);
                fast::st_async4(dst + 16, r.G, rbar);
                fast::st_async4(dst + 32, make_float4(r.M.x, r.M.y, 0.f, 0.f), rbar);
            }
            if (l == 0) fast::mbar_wait_cluster_bounded(&S.xbar, p.err);
            __syncwarp();
            // lanes as peers: rescale to the column maximum, scan across CTAs
            float2 Mr = f2(-INFINITY);
            float4 PF = fast::zero4(), PG = fast::zero4();
            if (l < p.ncl) {
                const Rec& r = S.mb[l][jj];
                Mr = r.M;
                PF = r.F;
                PG = r.G;
            }
            float2 Mc = Mr;
#pragma unroll
            for (int d = 1; d < kClusterMax; d <<= 1) {
                Mc.x = fmaxf(Mc.x, __shfl_xor_sync(0xffffffffu, Mc.x, d, kClusterMax));
                Mc.y = fmaxf(Mc.y, __shfl_xor_sync(0xffffffffu, Mc.y, d, kClusterMax));
            }
            // every lane of the warp needs lanes 0..7's column maximum
            Mc = make_float2(__shfl_sync(0xffffffffu, Mc.x, 0), __shfl_sync(0xffffffffu, Mc.y, 0));
            const float2 sc = make_float2(Mr.x == -INFINITY ? 0.f : ex2(Mr.x - Mc.x),
                                          Mr.y == -INFINITY ? 0.f : ex2(Mr.y - Mc.y));
            PF = scale4(sc, PF);
            PG = scale4(sc, PG);
#pragma unroll
            for (int e = 0; e < 3; ++e) {
                const int d = 1 << e;
                const float2 m = S.acl[e][jj];  // a^(512 d)
                const float4 uF = fast::shfl_up4(PF, d, kClusterMax);
                const float4 dG = fast::shfl_down4(PG, d, kClusterMax);
                if ((l & 7) >= d) PF = fma4(m, uF, PF);
                if ((l & 7) + d < kClusterMax) PG = fma4(m, dG, PG);
            }
            float4 colF = shfl_idx4(PF, rank > 0 ? rank - 1 : 0);
            float4 colG = shfl_idx4(PG, rank + 1 < p.ncl ? rank + 1 : 0);
            if (rank == 0) colF = fast::zero4();
            if (rank + 1 >= p.ncl) colG = fast::zero4();
            // column frame -> this CTA's frame: 2^(Mc - Mcta), exponent capped
            const float2 Mown = make_float2(__shfl_sync(0xffffffffu, Mr.x, rank),
                                            __shfl_sync(0xffffffffu, Mr.y, rank));
            const float2 up = make_float2(Mown.x == -INFINITY ? 0.f : ex2(fminf(Mc.x - Mown.x, kCarryExpCap)),
                                          Mown.y == -INFINITY ? 0.f : ex2(fminf(Mc.y - Mown.y, kCarryExpCap)));
            colF = scale4(up, colF);
            colG = scale4(up, colG);
            if (SEG) {
                // this segment's totals (frame Mc): forward at the last peer,
                // backward at the first; published by the cluster's rank 0
                const float4 sF = shfl_idx4(PF, p.ncl - 1), sG = shfl_idx4(PG, 0);
                const size_t cs = (size_t)col * p.nseg;
                if (rank == 0 && l == 0) {
                    float4* rec = p.ws_rec + ((cs + seg) * kNP + jj) * 3;
                    __stcg(rec, sF);
                    __stcg(rec + 1, sG);
                    __stcg(rec + 2, make_float4(Mc.x, Mc.y, 0.f, 0.f));
                    __threadfence();
                }
                __syncthreads();  // every pair's record is out
                if (rank == 0 && tid == 0)
                    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.ws_flag + cs + seg), "r"(gen + 1u)
                                 : "memory");
                // lanes as segments: wait for the column's records, rescale to
                // the column maximum, scan across segments
                float2 Ms = f2(-INFINITY);
                float4 SF = fast::zero4(), SG = fast::zero4();
                if (l < p.nseg) {
                    wait_flag_bounded(p.ws_flag + cs + l, gen + 1u, p.err);
                    const float4* rec = p.ws_rec + ((cs + l) * kNP + jj) * 3;
                    SF = __ldcg(rec);
                    SG = __ldcg(rec + 1);
                    const float4 m4 = __ldcg(rec + 2);
                    Ms = make_float2(m4.x, m4.y);
                }
                float2 Mcol = Ms;
#pragma unroll
                for (int d = 1; d < 8; d <<= 1) {
                    Mcol.x = fmaxf(Mcol.x, __shfl_xor_sync(0xffffffffu, Mcol.x, d, 8));
                    Mcol.y = fmaxf(Mcol.y, __shfl_xor_sync(0xffffffffu, Mcol.y, d, 8));
                }
                Mcol = make_float2(__shfl_sync(0xffffffffu, Mcol.x, 0), __shfl_sync(0xffffffffu, Mcol.y, 0));
                const float2 ss = make_float2(Ms.x == -INFINITY ? 0.f : ex2(Ms.x - Mcol.x),
                                              Ms.y == -INFINITY ? 0.f : ex2(Ms.y - Mcol.y));
                SF = scale4(ss, SF);
                SG = scale4(ss, SG);
#pragma unroll
                for (int e = 0; e < 3; ++e) {
                    const int d = 1 << e;
                    const float2 m = S.aseg[e][jj];  // a^(512 ncl d)
                    const float4 uF = fast::shfl_up4(SF, d, 8);
                    const float4 dG = fast::shfl_down4(SG, d, 8);
                    if ((l & 7) >= d) SF = fma4(m, uF, SF);
                    if ((l & 7) + d < 8) SG = fma4(m, dG, SG);
                }
                float4 gF = shfl_idx4(SF, seg > 0 ? seg - 1 : 0);
                float4 gG = shfl_idx4(SG, seg + 1 < p.nseg ? seg + 1 : 0);
                if (seg == 0) gF = fast::zero4();
                if (seg + 1 >= p.nseg) gG = fast::zero4();
                // column frame -> this CTA's frame, then decay to the CTA's ends:
                // forward from token 512 ncl seg - 1 to 512 grank - 1,
                // backward from token 512 ncl (seg + 1) to 512 (grank + 1)
                const float2 lam = mul2(make_float2(__ldg(p.w + c0 + 2 * jj), __ldg(p.w + c0 + 2 * jj + 1)),
                                        f2(p.invT * kLog2e));
                const float2 dF = ex2c(mul2(lam, f2(-(float)kTc * (float)rank)));
                const float2 dG = ex2c(mul2(lam, f2(-(float)kTc * (float)(p.ncl - 1 - rank))));
                const float2 up2 = make_float2(Mown.x == -INFINITY ? 0.f : ex2(fminf(Mcol.x - Mown.x, kCarryExpCap)),
                                               Mown.y == -INFINITY ? 0.f : ex2(fminf(Mcol.y - Mown.y, kCarryExpCap)));
                colF = fma4(mul2(up2, dF), gF, colF);
                colG = fma4(mul2(up2, dG), gG, colG);
            }
            // into chunk l: forward from token 512 r - 1 to 512 r + 16 l - 1,
            // backward from token 512 (r + 1) to 512 r + 16 (l + 1)
            cF = fma4(S.pw16[l][jj], colF, cF);
            cG = fma4(S.pw16[31 - l][jj], colG, cG);
        }
        S.aggF[l][jj] = cF;
        S.aggG[l][jj] = cG;
    }
    __syncthreads();

    // ---- 5. outputs: per sub-chunk a forward walk from the carry, then a
    // backward walk that finishes num and den ---------------------------------
    {
        const float4 cF = S.aggF[q][j], cG = S.aggG[q][j];
        const float2 eu = S.eu[j];
        // sub-chunk carries: h = 0 takes the chunk's forward carry and, from
        // the right, sub-chunk 1's total plus the chunk's backward carry;
        // h = 1 the reverse
        const float4 A0 = cF, B1 = cG;
        const float4 A1 = fma4(a8, cF, Fs[0]);
        const float4 B0 = fma4(a8, cG, Gs[1]);
        char* tout = const_cast<char*>(tb[0]);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float4 Ac = h == 0 ? A0 : A1, Bc = h == 0 ? B0 : B1;
            float2 A = fast::lo2(Ac), Cd = fast::hi2(Ac);
            float2 Y[kS], Z[kS];
#pragma unroll
            for (int i = 0; i < kS; ++i) {
                const int t = h * kS + i;
                Y[i] = fma2(eu, vv[t], A);
                Z[i] = fma2(eu, kk[t], Cd);
                A = fma2(alpha, A, vv[t]);
                Cd = fma2(alpha, Cd, kk[t]);
            }
            float2 Bn = fast::lo2(Bc), Dn = fast::hi2(Bc);
#pragma unroll
            for (int i = kS - 1; i >= 0; --i) {
                const int t = h * kS + i;
                const float2 num = add2(Y[i], Bn);
                float2 den = add2(Z[i], Dn);
                Bn = fma2(alpha, Bn, vv[t]);
                Dn = fma2(alpha, Dn, kk[t]);
                if (GATE) den = fma2(den, mypark[t * park_stride], den);
                st2<IO>(tout + t * RB, mul2(num, rcp(den)));
            }
        }
    }
    __syncthreads();

    // ---- coalesced copy-out of the results (first tile) ----------------------
    {
        constexpr int UPR = RB / 16;  // 16-byte units per token row
        const int ntok = min(kTc, p.T - t0);
        const char* tile0 = tiles + hb4 * CB;
        char* gout = p.out + ((size_t)b * p.T + t0) * p.C * es + (size_t)c0 * es;
        for (int u = tid; u < kTc * UPR; u += kThreads) {
            const int t = u / UPR, part = u - t * UPR;
            if (t < ntok)
                *reinterpret_cast<uint4*>(gout + (size_t)t * p.C * es + part * 16) =
                    *reinterpret_cast<const uint4*>(tile0 + (t / kL) * CB + (t % kL) * RB + part * 16);
        }
    }
    // no closing cluster barrier: every peer's record arrived in this CTA's
    // mailbox before its wait ended, and no CTA touches another's memory after
    if (SEG && tid == 0) {
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

}  // namespace wide
}  // namespace vrwkv
