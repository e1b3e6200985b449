// Fused Q-Shift -> Bi-WKV -> sigma(R) gate, TMA fast path for sm_100a.
//
// Same chunked two-sided scan as the generic kernel (biwkv.cuh) evaluating
// Bi-WKV of "Vision-RWKV Backbone", Linear Complexity Bidirectional
// Attention, eq. 5, on inputs Q-Shifted per Quad-Directional Token Shift,
// eq. 9, gated per Overall Architecture, eq. 2:
//
//   A_t = sum_{i<t} a^{t-1-i} p_i v_i,  B_t = sum_{i>t} a^{i-t-1} p_i v_i,
//   C_t, D_t with v = 1,  a = e^{-w/T},  p_i = e^{k_i - M},
//   wkv_t = (A_t + B_t + e^u p_t v_t) / (C_t + D_t + e^u p_t).
//
// Work decomposition: a CTA owns batch row b, a slab of kCS = 8 channels
// and 512 tokens; a thread owns one channel pair and a chunk of KL tokens
// (16 by default: two 8-token sub-chunks walked one after the other; 8
// where a cluster's CTAs cannot hold whole 128-token warps).  Each sub-chunk
// works relative to its own maximum of k, and the thread, warp, CTA and
// cluster steps rescale by 2^(M_lower - M_upper) <= 1 on the way up.
//
// What makes this path fast:
//  * Tiles arrive by TMA (cp.async.bulk.tensor, no multicast) with an element
//    stride of 8 along the token axis: box i (i = 0..7) holds tokens 8m + i,
//    so sub-tile i, row m is token i of sub-chunk m.  At each step the
//    sub-chunks a warp reads are consecutive rows (every other row with
//    16-token chunks), and every address is a compile-time offset from one
//    base register.
//  * With Q-Shift the (B, T, C) tensor is described as the 4-D image
//    (C, W, H, B) (W a multiple of 8, at most 256); the shifted tile x_shift
//    is the same set of boxes displaced by +-s along w or h.  TMA fills
//    out-of-image elements with zeros, which is exactly Q-Shift's zero
//    border, so no per-token shift arithmetic remains: token t of both tiles
//    sits at the same shared-memory offset.  Any other W takes the flat
//    token view: the shifted tile is displaced by the group's token offset
//    and its row-wrapped tokens are cleared after the load (zero_row_wrap).
//    A CTA's kCS channels lie in one channel group (the host requires the
//    group bounds to be multiples of kCS).
//  * Columns of at most 256 tokens (a 14 x 14 grid: 196) run 64-thread CTAs
//    of 256 tokens; longer ones 128-thread CTAs of 512.
//  * Four CTAs per SM (128 threads at <= 128 registers, or 256 at 64), so
//    one CTA's barriers and scans overlap another's arithmetic.  Sequences
//    longer than 512 tokens split over a thread-block cluster along T (8
//    CTAs at T = 4096: two SMs per cluster, so clusters fill every SM); CTA
//    aggregates travel by asynchronous stores into the peers' shared-memory
//    mailboxes that complete on the receiver's mbarrier.
//  * Results go back into the first input tile and leave by TMA tensor
//    stores in the same strided layout.
//  * Arrays that a warp reads down a column ([pair][warp], [peer][pair])
//    have one element of row padding, so those reads are bank-conflict free.
//  * Decay powers a^(KL m) come from a per-CTA table (one exp2 each), the
//    bf16 unpack is integer arithmetic, and arithmetic is packed float2.
// Exponents are base 2 (log2 e is folded into k, u, w and r).
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace vrwkv {
namespace fast {

constexpr int kCS = 8;          // channels per CTA (a column slab)
constexpr int kNP = kCS / 2;    // channel pairs per CTA
constexpr int kL = 8;           // tokens per sub-chunk (= the TMA element stride)
constexpr int kCPW = 32 / kNP;  // chunks per warp
constexpr int kClusterMax = 16;

// Limit of every bounded wait in the library's kernels, in nanoseconds of the
// GPU's global timer: 2 s unless vrwkv_set_wait_limit changes it (per device).
// A wait that runs out records a flag in the device error word and lets the
// kernel finish, so the context stays usable.
__device__ unsigned long long g_vrwkv_wait_ns = 2000000000ull;
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// CTA shape: NT threads = kNP channel pairs x NT/kNP chunks of KL tokens
// (KL = 8: one sub-chunk, 64 registers per thread; KL = 16: two sub-chunks
// of 8, 128 registers).  The library launches NT = 256 with KL = 8 and
// NT = 128 with KL = 16: both span 512 tokens, four CTAs per SM, clusters of
// up to 16 CTAs along T.
template <int NT, int KL>
struct Cfg {
    static_assert(KL == 8 || KL == 16, "8 or 16 tokens per thread chunk");
    static constexpr int kThreads = NT;
    static constexpr int kNW = NT / 32;             // warps
    static constexpr int kH = KL / kL;              // sub-chunks per chunk
    static constexpr int kTcMax = NT / kNP * KL;    // tokens per CTA
    static constexpr int kTab = kTcMax / KL;        // chunks per CTA: a^(KL m), m < kTab
    static constexpr int kWarpTok = kCPW * KL;      // tokens per warp
    static constexpr int kMinBlocks = 65536 / (NT * 16 * KL / 2);  // 64 or 128 registers per thread
};

enum Layout { kKV = 0, kRKV = 1, kX = 2 };

struct alignas(64) Params {
    CUtensorMap map[3];  // one per distinct source tensor (tile order below)
    CUtensorMap omap;    // the output, in the tiles' layout (stores by TMA)
    const float* w;
    const float* u;
    const float* mu[3];  // mu of r, k, v (each nullable)
    char* out;
    unsigned int* err;   // device error word (bounded waits)
    int B, T, C;
    int H, W, s;         // Q-Shift grid, shift
    QsBounds g;          // Q-Shift channel-group bounds (multiples of kCS on this path)
    int ng;              // shifted groups: 4 (Q-Shift) or 2 (bidirectional shift)
    float invT;          // 1 / T
    int Tc;              // tokens per CTA (multiple of kWarpTok when ncl > 1)
    int rows;            // image rows per CTA (Q-Shift path): Tc = rows * W
    int ncl;             // CTAs per column (cluster size)
    int tile_bytes;      // bytes per tile: 8 sub-tiles of 32 token rows
    int box_bytes;       // bytes one strided box delivers (zero fill included)
    int tma_store;       // results leave by TMA stores (the CTA's span is whole boxes, or the column's end)
    int flat;            // Q-Shift through the flat (C, T, B) view: shifted tiles loaded at a token
                         // offset, row-wrapped tokens of horizontal groups zeroed after the load
    // tensor-memory kernel only:
    int nbox;            // boxes per lane and tile (1 or 4); box g holds warps g * 4 / nbox onwards
                         // and completes on their tile barrier g
    int imaj;            // map[] are residue-major views (one box fills a whole tile, sub-tile i
                         // holding the tokens 8 m + i); xmap[] are the lane-strided views of the
                         // shifted tiles that a single box cannot displace
    int ofold;           // omap is the residue-major view: one store writes the CTA's results
    CUtensorMap xmap[3];
    // global-memory exchange (GX kernels only): see the workspace layout below
    unsigned int* ws_ctl;   // [0] ticket counter, [1] finished CTAs, [2] generation
    unsigned int* ws_flag;  // per (column, rank): generation + 1 once its record is out
    float4* ws_rec;         // per (column, rank): kRecF4 float4 record
    int nslab;           // channel slabs (C / 8)
    int total;           // CTAs in the grid
};

// Global-memory exchange.  Without clusters, the CTAs of one column find
// each other through a workspace: every CTA takes a ticket from a counter,
// tickets map column by column onto (rank, slab, b), so the <= 16 CTAs of a
// column hold consecutive tickets; a CTA publishes its aggregates (a record
// and a flag tagged with the launch's generation) and waits, with a bounded
// spin, for the flags of its column's peers.  Tickets are taken in start
// order, so the peers a CTA waits for have either started or start as soon
// as any CTA of an earlier, complete column exits: waiting can only stall a
// column that has not been fully started, and a GPU that holds 16 CTAs at once
// always starts it.  The last CTA to finish resets the counters and advances
// the generation, so stale flags of earlier launches never match.
constexpr int kRecF4 = 2 * kNP + kNP / 2;  // float4 per record: F, G per pair; M two pairs per float4

template <int NT, int KL>
struct alignas(16) Scratch {
    static constexpr int kNW = Cfg<NT, KL>::kNW;
    float2 tab[Cfg<NT, KL>::kTab][kNP];  // a^(KL m) per channel pair
    // Rows of the [pair][warp] and [peer][pair] arrays carry one element of
    // padding: a warp reads one column across eight (or sixteen) rows, and
    // the odd row stride spreads those reads over all 32 banks.
    float2 wmax[kNP][kNW + 1];      // per-warp maxima of k (-inf for a warp wholly past T)
    float2 wsc[kNP][kNW + 1];       // per-warp scale 2^(M_warp - M_cta) onto the CTA reference
    float4 waggF[kNP][kNW + 1];     // per-warp forward aggregates (A.xy, C.xy)
    float4 waggB[kNP][kNW + 1];     // per-warp backward aggregates
    float4 wcarF[kNP][kNW + 1];     // exclusive forward carry into each warp
    float4 wcarB[kNP][kNW + 1];     // exclusive backward carry into each warp
    float2 mbM[kClusterMax][kNP + 1];   // mailbox: each CTA's max of k (times log2 e)
    float4 mbF[kClusterMax][kNP + 1];   // mailbox: each CTA's forward aggregate
    float4 mbG[kClusterMax][kNP + 1];   // mailbox: each CTA's backward aggregate
    float4 ownF[kNP];           // this CTA's inclusive forward aggregate, staged for the push
    float4 ownG[kNP];           // this CTA's inclusive backward aggregate
    float2 ownM[kNP];           // this CTA's max of k (times log2 e)
    float4 cscale[kCS];         // per channel: sl (scale of this CTA's own sums)
    int tk;                     // GX: this CTA's ticket
    unsigned int gen;           // GX: the launch's generation
    float4 ccarry[kCS];         // per channel: carries Af, Cf, Bb, Db
    unsigned long long bar;     // TMA completion barrier
    unsigned long long xbar;    // mailbox barrier: completes when every peer's record is in
};

// Q-Shift through the flat token view (any W): a shifted tile loaded at the
// token offset -s or +s (horizontal groups 0 and 1) holds, at the first or
// last s columns of every image row, a token of the neighbouring row.  eq. 9
// wants zeros there; this clears those token rows of each source's shifted
// tile (tile 2 src + 1) after the load.  Vertical groups need nothing: the
// offset -s W or +s W leaves [0, T) exactly where the row leaves [0, H), and
// the TMA's zero fill covers it.  Token tl of the CTA sits at sub-tile tl % 8,
// row tl / 8.
// The tokens cleared are those in [lo, hi); t0 is the CTA's first token.
// Threads take image rows; one division per thread.
template <int RB>
__device__ __forceinline__ void zero_row_wrap(char* smem, int tile_bytes, int sub_bytes, int nsrc, int t0, int lo,
                                              int hi, int W, int s, bool left, int tid, int nthreads) {
    if (hi <= lo) return;
    const int sw = min(s, W);  // source outside the row: w < s (left) or w >= W - s
    for (int hr = lo / W + tid, t_row = hr * W; t_row < hi; hr += nthreads, t_row += nthreads * W) {
        for (int k = 0; k < sw; ++k) {
            const int t = t_row + (left ? k : W - 1 - k);
            if (t < lo || t >= hi) continue;
            const int tl = t - t0;
            for (int src = 0; src < nsrc; ++src) {
                char* dst = smem + (2 * src + 1) * tile_bytes + (tl & (kL - 1)) * sub_bytes + (tl / kL) * RB;
#pragma unroll
                for (int o = 0; o < RB; o += 16) *reinterpret_cast<uint4*>(dst + o) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
    }
}

// One float of a tile slot: the gate factor parked between the load and the
// output pass (see the kernels).  A gate factor's store into a slot depends
// on the values read from that slot (they make r), and a result's store on
// the gate factor read from its slot: data dependence alone orders each
// slot's accesses.
__device__ __forceinline__ void sts_f32(char* p, float v) { *reinterpret_cast<float*>(p) = v; }
__device__ __forceinline__ float lds_f32(const char* p) { return *reinterpret_cast<const float*>(p); }

// ---- PTX wrappers ----------------------------------------------------------
__device__ __forceinline__ unsigned smem_u32(const void* p) {
    return (unsigned)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(unsigned long long* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// try_wait with a suspend-time hint (ns): the thread sleeps in hardware until
// the phase completes or the hint elapses, instead of spinning.
__device__ __forceinline__ bool mbar_try_wait(unsigned long long* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
// Wait for phase 0 of the barrier; give up after the wait limit, record the
// failure in the device error word and continue (the caller's barriers stay
// matched).
__device__ __forceinline__ void mbar_wait_bounded(unsigned long long* bar, unsigned* err) {
    if (mbar_try_wait(bar, 0)) return;
    const unsigned long long t0 = global_ns(), lim = g_vrwkv_wait_ns;
    while (!mbar_try_wait(bar, 0)) {
        if (global_ns() - t0 > lim) {
            atomicOr(err, 1u);
            return;
        }
    }
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_u32(bar))
        : "memory");
}
// Store a box of a shared-memory tile to global memory (bulk async group);
// elements outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<unsigned long long>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            int c3, int c4, unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<unsigned long long>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit_and_wait_read() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA) of this CTA.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ unsigned mapa_u32(unsigned a, unsigned rank) {
    unsigned r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    return r;
}
// Asynchronous store into another CTA's shared memory that completes its
// bytes on that CTA's mbarrier (no fence, no cluster barrier).
__device__ __forceinline__ void st_async4(unsigned raddr, float4 v, unsigned rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(raddr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(rbar) : "memory");
}
__device__ __forceinline__ void st_async2(unsigned raddr, float2 v, unsigned rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];"
                 ::"r"(raddr), "f"(v.x), "f"(v.y), "r"(rbar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(unsigned long long* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_wait_cluster_bounded(unsigned long long* bar, unsigned* err) {
    if (mbar_try_wait_cluster(bar, 0)) return;
    const unsigned long long t0 = global_ns(), lim = g_vrwkv_wait_ns;
    while (!mbar_try_wait_cluster(bar, 0)) {
        if (global_ns() - t0 > lim) {
            atomicOr(err, 1u);
            return;
        }
    }
}
__device__ __forceinline__ void cluster_wait_acquire() {
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Channel pair of one token from a tile, as float2.
template <typename IO>
__device__ __forceinline__ float2 lds_pair(const char* tile, int off);
template <>
__device__ __forceinline__ float2 lds_pair<__nv_bfloat16>(const char* tile, int off) {
    const unsigned u = *reinterpret_cast<const unsigned*>(tile + off);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
template <>
__device__ __forceinline__ float2 lds_pair<float>(const char* tile, int off) {
    return *reinterpret_cast<const float2*>(tile + off);
}

__device__ __forceinline__ float4 shfl_up4(float4 v, int d, int width) {
    return make_float4(__shfl_up_sync(0xffffffffu, v.x, d, width), __shfl_up_sync(0xffffffffu, v.y, d, width),
                       __shfl_up_sync(0xffffffffu, v.z, d, width), __shfl_up_sync(0xffffffffu, v.w, d, width));
}
__device__ __forceinline__ float4 shfl_down4(float4 v, int d, int width) {
    return make_float4(__shfl_down_sync(0xffffffffu, v.x, d, width),
                       __shfl_down_sync(0xffffffffu, v.y, d, width),
                       __shfl_down_sync(0xffffffffu, v.z, d, width),
                       __shfl_down_sync(0xffffffffu, v.w, d, width));
}
__device__ __forceinline__ float4 fma4(float2 m, float4 x, float4 y) {
    const float2 a = fma2(m, make_float2(x.x, x.y), make_float2(y.x, y.y));
    const float2 c = fma2(m, make_float2(x.z, x.w), make_float2(y.z, y.w));
    return make_float4(a.x, a.y, c.x, c.y);
}
__device__ __forceinline__ float2 lo2(float4 v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(float4 v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float4 zero4() { return make_float4(0.f, 0.f, 0.f, 0.f); }

// Bounded wait for a peer's flag (acquire); records a timeout in the device
// error word (bit 1) and gives up instead of hanging.
__device__ __forceinline__ void wait_flag(const unsigned int* f, unsigned int want, unsigned int* err) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    if (v == want) return;
    const unsigned long long t0 = global_ns(), lim = g_vrwkv_wait_ns;
    unsigned int ns = 32;
    for (;;) {
        __nanosleep(ns);
        if (ns < 1024) ns <<= 1;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
        if (v == want) return;
        if (global_ns() - t0 > lim) {
            atomicOr(err, 2u);
            return;
        }
    }
}

template <typename IO, int LAYOUT, bool QS, int NT, int KL, bool GX>
__global__ void __launch_bounds__(NT, Cfg<NT, KL>::kMinBlocks)
    biwkv_tma_kernel(const __grid_constant__ Params p) {
    using C_ = Cfg<NT, KL>;
    constexpr int kThreads = C_::kThreads;
    constexpr int kNW = C_::kNW;
    constexpr int kTcMax = C_::kTcMax;
    constexpr int kH = C_::kH;          // sub-chunks of 8 tokens per thread chunk
    using Scratch = fast::Scratch<NT, KL>;
    constexpr bool GATE = LAYOUT != kKV;
    constexpr int NSRC = LAYOUT == kKV ? 2 : (LAYOUT == kRKV ? 3 : 1);
    constexpr int NTILE = NSRC * (QS ? 2 : 1);
    constexpr int SR = 0;
    constexpr int SK = LAYOUT == kRKV ? 1 : 0;
    constexpr int SV = LAYOUT == kKV ? 1 : (LAYOUT == kRKV ? 2 : 0);
    constexpr int es = Io<IO>::kBytes;
    constexpr int RB = kCS * es;  // bytes per token row of a tile
    constexpr int PB = 2 * es;    // bytes per channel pair

    // dynamic shared memory, re-aligned to 128 bytes for the TMA
    // destinations; the host adds 128 bytes of slack
    extern __shared__ __align__(128) char smem_raw[];
    char* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    // The gate factor e^{-r} of a token waits for the output pass in two tile
    // slots its thread has just read: r's own and shifted r's with Q-Shift;
    // r's and k's for separate r, k, v without; r's and one extra tile when
    // one x feeds r, k and v without Q-Shift.  The result later goes into the
    // first slot.
    constexpr bool G1_IN_K = GATE && !QS && LAYOUT == kRKV;
    constexpr int NTA = GATE && !QS && !G1_IN_K ? NTILE + 1 : NTILE;
    constexpr int G1 = QS ? 2 * SR + 1 : (G1_IN_K ? SK : NTILE);  // tile of the second half
    Scratch& S = *reinterpret_cast<Scratch*>(smem + NTA * p.tile_bytes);

    const int tid = threadIdx.x;
    const int j = tid % kNP;     // channel pair
    const int q = tid / kNP;     // chunk within the CTA
    const int cq = q % kCPW;     // chunk within the warp
    const int warp = tid >> 5;
    if (tid == 0) {
        mbar_init(&S.bar, 1);
        if (!GX && p.ncl > 1) {
            // the mailbox barrier: one arrival (here) plus every peer's bytes
            mbar_init(&S.xbar, 1);
            mbar_expect_tx(&S.xbar, (unsigned)(p.ncl * kNP * (sizeof(float4) * 2 + sizeof(float2))));
        }
        if (GX) {
            S.tk = (int)atomicAdd(p.ws_ctl, 1u);
            S.gen = *reinterpret_cast<volatile unsigned int*>(p.ws_ctl + 2);
        }
    }
    __syncthreads();
    // mailbox barriers initialised cluster-wide before anyone pushes: arrive
    // now, wait just before the first push
    if (!GX && p.ncl > 1) cluster_arrive_relaxed();
    // this CTA's column chunk: the block index, or (GX) the ticket
    int rank = blockIdx.x, slab = blockIdx.y, b = blockIdx.z;
    unsigned int gen = 0;
    if (GX) {
        const int t = S.tk;
        if (t < 0 || t >= p.total) {  // a workspace that was not zero-filled
            if (tid == 0) atomicOr(p.err, 4u);
            return;
        }
        gen = S.gen;
        rank = t % p.ncl;
        slab = (t / p.ncl) % p.nslab;
        b = t / p.ncl / p.nslab;
    }
    const int col = b * p.nslab + slab;  // GX: the column's records and flags
    const int c0 = slab * kCS;
    const int t0 = rank * p.Tc;
    const int tend = min(p.T, t0 + p.Tc);

    // group of this CTA's channels (Q-Shift): 0..3 shifted, 4 copied
    int grp = QS ? qs_group(c0, p.g) : 4;
    if (grp >= p.ng) grp = 4;
    const bool shifted = QS && grp < 4;

    // ---- issue the tile loads: lane i of warp 0 loads sub-tile i of each tile
    constexpr int SUB = kTcMax / kL * RB;  // bytes per sub-tile (kTcMax / 8 token rows)
    if (warp == 0) {
        if (tid == 0) {
            mbar_expect_tx(&S.bar, (unsigned)p.box_bytes * (unsigned)(kL * NSRC * (shifted ? 2 : 1)));
        }
        __syncwarp();
        if (tid < kL) {
            const int i = tid;
            const int h0 = rank * p.rows;
            for (int s = 0; s < NSRC; ++s) {
                char* plain = smem + (QS ? 2 * s : s) * p.tile_bytes + i * SUB;
                if (!QS || p.flat) {
                    // boxes of 256 strided tokens (32 rows); a box wholly past T
                    // still delivers its zero-filled bytes
#pragma unroll
                    for (int h = 0; h < kTcMax / 256; ++h)
                        tma_load_3d(plain + h * 32 * RB, &p.map[s], c0, t0 + i + 256 * h, b, &S.bar);
                    if (QS && shifted) {
                        // the flat view: the same boxes displaced by the group's token offset
                        const int dt = grp == 0 ? -p.s : (grp == 1 ? p.s : (grp == 2 ? -p.s * p.W : p.s * p.W));
#pragma unroll
                        for (int h = 0; h < kTcMax / 256; ++h)
                            tma_load_3d(plain + p.tile_bytes + h * 32 * RB, &p.map[s], c0, t0 + i + dt + 256 * h, b,
                                        &S.bar);
                    }
                } else {
                    tma_load_4d(plain, &p.map[s], c0, i, h0, b, &S.bar);
                    if (shifted) {
                        const int dw = grp == 0 ? -p.s : (grp == 1 ? p.s : 0);
                        const int dh = grp == 2 ? -p.s : (grp == 3 ? p.s : 0);
                        tma_load_4d(plain + p.tile_bytes, &p.map[s], c0, i + dw, h0 + dh, b, &S.bar);
                    }
                }
            }
        }
    }

    // ---- per-thread constants (overlap the copies) ---------------------------
    const int cA = c0 + 2 * j;
    const float invT = p.invT;
    const float2 wv = make_float2(__ldg(p.w + cA), __ldg(p.w + cA + 1));
    const float2 uv = make_float2(__ldg(p.u + cA), __ldg(p.u + cA + 1));
    const float2 lam2 = mul2(wv, f2(invT * kLog2e));  // w / T in base-2 units
    const float2 alpha = ex2c(make_float2(-lam2.x, -lam2.y));
    const float2 eu = ex2(mul2(uv, f2(kLog2e)));
    const float2 a8 = ex2c(mul2(lam2, f2(-(float)kL)));  // a^8: across one sub-chunk (KL = 16)
    auto mu_of = [&](const float* m) {
        return m ? make_float2(__ldg(m + cA), __ldg(m + cA + 1)) : f2(0.0f);
    };
    const float2 muk = QS ? mu_of(p.mu[1]) : f2(1.0f);
    const float2 muv = QS ? mu_of(p.mu[2]) : f2(1.0f);
    const float2 mur = (QS && GATE) ? mu_of(p.mu[0]) : f2(1.0f);
    // decay table a^(KL m), one per chunk distance m: one entry (2 channels)
    // per thread
    {
        const int m = tid / kNP, jj = tid % kNP;
        const float2 l = mul2(make_float2(__ldg(p.w + c0 + 2 * jj), __ldg(p.w + c0 + 2 * jj + 1)),
                              f2(invT * kLog2e));
        S.tab[m][jj] = ex2c(mul2(l, f2(-(float)KL * m)));
    }

    const int s_tok = t0 + q * KL;
    const int nvt = max(0, min(KL, tend - s_tok));  // valid tokens of this chunk

    // one thread waits for the tiles; the others sleep at the CTA barrier
    if (tid == 0) mbar_wait_bounded(&S.bar, p.err);
    __syncthreads();
    if (QS && p.flat && shifted && grp < 2) {
        zero_row_wrap<RB>(smem, p.tile_bytes, SUB, NSRC, t0, t0, tend, p.W, p.s, grp == 0, tid, kThreads);
        __syncthreads();
    }

    // ---- 1-2. per 8-token sub-chunk: load, Q-Shift mix, gate factor, local
    // maximum, p = 2^(k - M_h), two-sided sums inside the sub-chunk ----------
    // Token 8 (q kH + h) + i of the CTA is sub-tile i, row q kH + h.  Each
    // sub-chunk works relative to its own maximum M_h (0 if it lies wholly past
    // T); the thread combine below rescales by 2^(M_h - M_warp) <= 1.
    const char* tK = smem + (QS ? 2 * SK : SK) * p.tile_bytes;
    const char* tV = smem + (QS ? 2 * SV : SV) * p.tile_bytes;
    const char* tR = smem + (QS ? 2 * SR : SR) * p.tile_bytes;
    const int dsh = shifted ? p.tile_bytes : 0;  // shifted tile = plain + dsh
    // With 16-token chunks the lanes of chunks 4..7 of a warp take their two
    // sub-chunks in the opposite order: at each step the warp's eight chunks
    // read rows 2 q + (h ^ rot), eight different rows modulo 8, so tile, gate
    // and result accesses are free of bank conflicts.  Register arrays are
    // indexed by step; h is the sub-chunk a step works on.
    const int rot = kH == 2 ? (cq >> 2) & 1 : 0;
    float2 n[kH][kL], dd[kH][kL];
    float4 Fh[kH], Gh[kH];  // per step: forward (A.xy, C.xy) and backward totals of its sub-chunk
    float2 Mh[kH];          // per step: its sub-chunk's maximum of k (-inf if wholly past T)
#pragma unroll
    for (int st = 0; st < kH; ++st) {
        const int h = st ^ rot;
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
                    const float2 d = add2(x, make_float2(-xd.x, -xd.y));
                    k = fma2(muk, d, xd);
                    v = fma2(muv, d, xd);
                    r = fma2(mur, d, xd);
                } else {
                    const float2 xk = lds_pair<IO>(tK, o), xkd = lds_pair<IO>(tK + dsh, o);
                    const float2 xv = lds_pair<IO>(tV, o), xvd = lds_pair<IO>(tV + dsh, o);
                    k = fma2(muk, add2(xk, make_float2(-xkd.x, -xkd.y)), xkd);
                    v = fma2(muv, add2(xv, make_float2(-xvd.x, -xvd.y)), xvd);
                    if (GATE) {
                        const float2 xr = lds_pair<IO>(tR, o), xrd = lds_pair<IO>(tR + dsh, o);
                        r = fma2(mur, add2(xr, make_float2(-xrd.x, -xrd.y)), xrd);
                    }
                }
            } else {
                k = lds_pair<IO>(tK, o);
                v = lds_pair<IO>(tV, o);
                if (GATE) r = lds_pair<IO>(tR, o);
            }
            // gate factor e^{-r}, parked in the token's slots until the output pass
            if (GATE) {
                float2 g = ex2(mul2(r, f2(-kLog2e)));
                // in k's slot the second half must follow the read of k, which
                // it does not depend on: tie it to k (no instruction)
                if (G1_IN_K) asm volatile("" : "+f"(g.y) : "f"(k.x), "f"(k.y));
                sts_f32(smem + SR * (QS ? 2 : 1) * p.tile_bytes + o, g.x);
                sts_f32(smem + G1 * p.tile_bytes + o, g.y);
            }
            kk[i] = k;
            vv[i] = v;
        }
        float2 mx = f2(-INFINITY);
        if (nv == kL) {
#pragma unroll
            for (int i = 0; i < kL; ++i) mx = max2(mx, kk[i]);
        } else {
            // tokens past the sequence end hold zeros (TMA fill) or stale shared
            // memory (rows beyond a short box): mask both so p = 0 and p*v = 0
#pragma unroll
            for (int i = 0; i < kL; ++i) {
                kk[i] = (i < nv) ? kk[i] : f2(-INFINITY);
                vv[i] = (i < nv) ? vv[i] : f2(0.0f);
                mx = max2(mx, kk[i]);
            }
        }
        Mh[st] = mx;
        const float2 negM = make_float2(mx.x == -INFINITY ? 0.0f : -mx.x * kLog2e,
                                        mx.y == -INFINITY ? 0.0f : -mx.y * kLog2e);
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            kk[i] = ex2(fma2(kk[i], f2(kLog2e), negM));  // p_i (0 beyond T)
            vv[i] = mul2(kk[i], vv[i]);                  // p_i v_i
        }
        // Two-sided sums inside the sub-chunk, both directions in one walk
        // (four independent recurrences per step): step it adds the forward
        // sum before token it and the backward sum after token 7 - it; a
        // token's second contribution also brings its own term e^u p v.
        float2 fa = f2(0.0f), fc = f2(0.0f), ga = f2(0.0f), gc = f2(0.0f);
#pragma unroll
        for (int it = 0; it < kL; ++it) {
            const int i = it, ib = kL - 1 - it;
            if (it < kL / 2) {
                n[st][i] = fa;
                dd[st][i] = fc;
                n[st][ib] = ga;
                dd[st][ib] = gc;
            } else {
                n[st][i] = add2(n[st][i], fma2(eu, vv[i], fa));
                dd[st][i] = add2(dd[st][i], fma2(eu, kk[i], fc));
                n[st][ib] = add2(n[st][ib], fma2(eu, vv[ib], ga));
                dd[st][ib] = add2(dd[st][ib], fma2(eu, kk[ib], gc));
            }
            fa = fma2(alpha, fa, vv[i]);
            fc = fma2(alpha, fc, kk[i]);
            ga = fma2(alpha, ga, vv[ib]);
            gc = fma2(alpha, gc, kk[ib]);
        }
        Fh[st] = make_float4(fa.x, fa.y, fc.x, fc.y);
        Gh[st] = make_float4(ga.x, ga.y, gc.x, gc.y);
    }

    // ---- 3a. warp maximum (the reference of the warp's sums) and the chunk's
    // totals on it ---------------------------------------------------------------
    float2 mx = Mh[0];
#pragma unroll
    for (int st = 1; st < kH; ++st) mx = max2(mx, Mh[st]);
#pragma unroll
    for (int d = kNP; d < 32; d <<= 1) {
        mx.x = fmaxf(mx.x, __shfl_xor_sync(0xffffffffu, mx.x, d));
        mx.y = fmaxf(mx.y, __shfl_xor_sync(0xffffffffu, mx.y, d));
    }
    if (cq == 0) S.wmax[j][warp] = mx;  // -inf for a warp wholly past T
    // sub-chunk h -> warp reference: 2^(M_h - M_warp), 0 for an empty sub-chunk
    const float2 mref = make_float2(mx.x == -INFINITY ? 0.0f : mx.x, mx.y == -INFINITY ? 0.0f : mx.y);
    float2 eh[kH];
#pragma unroll
    for (int st = 0; st < kH; ++st) eh[st] = ex2(mul2(add2(Mh[st], make_float2(-mref.x, -mref.y)), f2(kLog2e)));
    auto scale4 = [](float2 e, float4 v) { return make_float4(v.x * e.x, v.y * e.y, v.z * e.x, v.w * e.y); };
    auto sel4 = [](bool c, float4 a, float4 b) { return c ? a : b; };
    float4 Fi, Gi;
    float4 F0s = zero4(), G1s = zero4();  // KL = 16: sub-chunk 0's forward, sub-chunk 1's backward total
    if (kH == 1) {
        Fi = scale4(eh[0], Fh[0]);
        Gi = scale4(eh[0], Gh[0]);
    } else {
        // sub-chunk 0 was step rot, sub-chunk 1 step 1 - rot
        const float4 sF0 = scale4(eh[0], Fh[0]), sF1 = scale4(eh[1], Fh[1]);
        const float4 sG0 = scale4(eh[0], Gh[0]), sG1 = scale4(eh[1], Gh[1]);
        F0s = sel4(rot, sF1, sF0);
        G1s = sel4(rot, sG0, sG1);
        Fi = fma4(a8, F0s, sel4(rot, sF0, sF1));
        Gi = fma4(a8, G1s, sel4(rot, sG1, sG0));
    }

    // ---- 3b. scans: warp, CTA, cluster -----------------------------------------
    // warp scan across the kCPW chunks of a warp: step e spans 2^e chunks
#pragma unroll
    for (int e = 0; (kNP << e) < 32; ++e) {
        const float2 m = S.tab[1 << e][j];  // a^(KL * 2^e)
        float4 o = shfl_up4(Fi, kNP << e, 32);
        if (cq >= (1 << e)) Fi = fma4(m, o, Fi);
        o = shfl_down4(Gi, kNP << e, 32);
        if (cq + (1 << e) < kCPW) Gi = fma4(m, o, Gi);
    }
    float4 X = shfl_up4(Fi, kNP, 32), Y = shfl_down4(Gi, kNP, 32);
    if (cq == 0) X = zero4();
    if (cq == kCPW - 1) Y = zero4();
    if (cq == kCPW - 1) S.waggF[j][warp] = Fi;
    if (cq == 0) S.waggB[j][warp] = Gi;
    __syncthreads();
    if (warp == 0) {  // lanes (pair, warp) < kNP * kNW; the rest idle along
        const bool act = tid < kNP * kNW;
        const int jj = act ? tid / kNW : 0, wi = act ? tid % kNW : 0;
        // CTA maximum; warp wi's sums move onto it by 2^(M_wi - M_cta) <= 1
        // (0 for a warp wholly past T)
        const float2 mw = S.wmax[jj][wi];
        float2 mc = mw;
#pragma unroll
        for (int d = 1; d < kNW; d <<= 1) {
            mc.x = fmaxf(mc.x, __shfl_xor_sync(0xffffffffu, mc.x, d, kNW));
            mc.y = fmaxf(mc.y, __shfl_xor_sync(0xffffffffu, mc.y, d, kNW));
        }
        const float2 ws = ex2(mul2(add2(mw, make_float2(-mc.x, -mc.y)), f2(kLog2e)));
        float4 f = scale4(ws, S.waggF[jj][wi]);
        float4 gb = scale4(ws, S.waggB[jj][wi]);
#pragma unroll
        for (int d = 1; d < kNW; d <<= 1) {
            const float2 m = S.tab[kCPW * d][jj];  // a^(KL kCPW d): across d warps
            float4 o = shfl_up4(f, d, kNW);
            if (wi >= d) f = fma4(m, o, f);
            o = shfl_down4(gb, d, kNW);
            if (wi + d < kNW) gb = fma4(m, o, gb);
        }
        float4 xw = shfl_up4(f, 1, kNW), yw = shfl_down4(gb, 1, kNW);
        if (wi == 0) xw = zero4();
        if (wi == kNW - 1) yw = zero4();
        if (act) {
            S.wsc[jj][wi] = ws;
            S.wcarF[jj][wi] = xw;
            S.wcarB[jj][wi] = yw;
            // stage this CTA's record; the CTA's forward aggregate sits at its
            // last real warp (Tc may be shorter than the CTA's capacity)
            if (p.ncl > 1) {
                if (wi == p.Tc / C_::kWarpTok - 1) S.ownF[jj] = f;
                if (wi == 0) {
                    S.ownG[jj] = gb;
                    S.ownM[jj] = mul2(mc, f2(kLog2e));  // base 2, the unit of the exponents below
                }
            }
        }
    }
    // Thread (peer rr, channel lc) of the exchange below: segments of sw
    // lanes, one per channel (8 lanes when the column has at most 8 CTAs, else
    // 16), so the first kCS * sw threads take part.  Decay powers across
    // d = 1, 2, 4 (, 8) CTAs are computed before the wait for the peers.
    const bool narrow = p.ncl <= 8;
    const int sw = narrow ? 8 : 16;
    const int lc = narrow ? tid >> 3 : tid >> 4, rr = tid & (sw - 1);
    const int nex = kCS * sw;  // a multiple of 32: warp-uniform
    float mdec[4];
    if (p.ncl > 1) {
        if (tid < nex) {
            const float l2 = __ldg(p.w + c0 + lc) * (invT * kLog2e);
#pragma unroll
            for (int e = 0; e < 4; ++e) mdec[e] = (1 << e) < sw ? ex2c(-(float)(p.Tc << e) * l2) : 0.0f;
        }
        __syncthreads();
        if (GX) {
            // publish the record to the workspace, then the flag (release
            // after every writer's fence), then wait for the column's flags
            // and copy the records into the mailbox
            float4* rec = p.ws_rec + ((size_t)col * kClusterMax + rank) * kRecF4;
            if (tid < kRecF4) {
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
            unsigned int* flags = p.ws_flag + (size_t)col * kClusterMax;
            if (tid == 0)
                asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(flags + rank), "r"(gen + 1u) : "memory");
            if (tid < p.ncl) wait_flag(flags + tid, gen + 1u, p.err);
            __syncthreads();
            const float4* peers = p.ws_rec + (size_t)col * kClusterMax * kRecF4;
            for (int e = tid; e < p.ncl * kRecF4; e += kThreads) {
                const int r = e / kRecF4, k = e - r * kRecF4;
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
        } else {
            // asynchronous stores of the record into every CTA's mailbox (its
            // own included), one (peer, pair, half) per thread, completing on
            // the receiver's mailbox barrier
            cluster_wait_acquire();  // every mailbox barrier is initialised
            const int peer = tid / (2 * kNP), jj = (tid >> 1) % kNP;
            if (peer < p.ncl) {
                const unsigned rbar = mapa_u32(smem_u32(&S.xbar), peer);
                if ((tid & 1) == 0) {
                    st_async4(mapa_u32(smem_u32(&S.mbF[rank][jj]), peer), S.ownF[jj], rbar);
                } else {
                    st_async4(mapa_u32(smem_u32(&S.mbG[rank][jj]), peer), S.ownG[jj], rbar);
                    st_async2(mapa_u32(smem_u32(&S.mbM[rank][jj]), peer), S.ownM[jj], rbar);
                }
            }
        }
    }
    if (p.ncl > 1 && !GX) {
        if (tid == 0) mbar_wait_cluster_bounded(&S.xbar, p.err);
        __syncthreads();
    } else {
        __syncthreads();
    }
    // Exchange with the other CTAs of the column: thread (channel lc, peer
    // rr) reads peer rr's record for channel lc from this CTA's mailbox;
    // each sw-lane segment holds one channel's column.  The segment maximum
    // of the peers' exponents is the common reference; forward and backward
    // carries are sw-lane shuffle scans with the one-CTA decay a^Tc.
    float2 cs_sl = f2(1.0f), cs_af = f2(0.0f), cs_cf = f2(0.0f), cs_bb = f2(0.0f), cs_db = f2(0.0f);
    if (p.ncl > 1) {
        if (tid < nex) {  // warp-uniform
            float Mr = -INFINITY, fa2 = 0.f, fc2 = 0.f, ga2 = 0.f, gc2 = 0.f;
            if (rr < p.ncl) {
                const float4 F = S.mbF[rr][lc >> 1], G = S.mbG[rr][lc >> 1];
                const float2 Mp = S.mbM[rr][lc >> 1];
                const bool hi = lc & 1;
                Mr = hi ? Mp.y : Mp.x;
                fa2 = hi ? F.y : F.x;
                fc2 = hi ? F.w : F.z;
                ga2 = hi ? G.y : G.x;
                gc2 = hi ? G.w : G.z;
            }
            float Mc = Mr;
#pragma unroll
            for (int d = 8; d >= 1; d >>= 1)
                if (d < sw) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, d, sw));
            const float sc = ex2(Mr - Mc);  // 0 for lanes past the cluster
            fa2 *= sc;
            fc2 *= sc;
            ga2 *= sc;
            gc2 *= sc;
#pragma unroll
            for (int e = 0, d = 1; d < kClusterMax; ++e, d <<= 1) {
                if (d >= sw) break;
                const float m = mdec[e];  // decay across d CTAs
                const float ua = __shfl_up_sync(0xffffffffu, fa2, d, sw);
                const float uc = __shfl_up_sync(0xffffffffu, fc2, d, sw);
                const float da = __shfl_down_sync(0xffffffffu, ga2, d, sw);
                const float dc = __shfl_down_sync(0xffffffffu, gc2, d, sw);
                if (rr >= d) {
                    fa2 = fmaf(m, ua, fa2);
                    fc2 = fmaf(m, uc, fc2);
                }
                if (rr + d < sw) {
                    ga2 = fmaf(m, da, ga2);
                    gc2 = fmaf(m, dc, gc2);
                }
            }
            // exclusive carries of this CTA: inclusive forward at rank-1,
            // inclusive backward at rank+1 (zero past the ends)
            const float Af = __shfl_sync(0xffffffffu, fa2, max(rank - 1, 0), sw);
            const float Cf = __shfl_sync(0xffffffffu, fc2, max(rank - 1, 0), sw);
            const float Bb = __shfl_sync(0xffffffffu, ga2, min(rank + 1, sw - 1), sw);
            const float Db = __shfl_sync(0xffffffffu, gc2, min(rank + 1, sw - 1), sw);
            const float Mme = __shfl_sync(0xffffffffu, Mr, rank, sw);
            if (rr == 0) {
                S.cscale[lc] = make_float4(ex2(Mme - Mc), 0.f, 0.f, 0.f);
                S.ccarry[lc] = make_float4(rank > 0 ? Af : 0.f, rank > 0 ? Cf : 0.f,
                                           rank + 1 < p.ncl ? Bb : 0.f, rank + 1 < p.ncl ? Db : 0.f);
            }
        }
        __syncthreads();
        const float4 s0 = S.cscale[2 * j], s1 = S.cscale[2 * j + 1];
        const float4 k0 = S.ccarry[2 * j], k1 = S.ccarry[2 * j + 1];
        cs_sl = make_float2(s0.x, s1.x);
        cs_af = make_float2(k0.x, k1.x);
        cs_cf = make_float2(k0.y, k1.y);
        cs_bb = make_float2(k0.z, k1.z);
        cs_db = make_float2(k0.w, k1.w);
    }

    // ---- 4. carries -> outputs ---------------------------------------------------
    // sl: CTA reference -> column reference; slw: this warp's reference ->
    // column reference (the warp-local sums X, Y and the sub-chunk totals use
    // the warp's own; n, dd use their sub-chunk's, hence the extra eh)
    const float2 sl = cs_sl;
    const float2 slw = mul2(sl, S.wsc[j][warp]);
    const float4 XW = S.wcarF[j][warp], YW = S.wcarB[j][warp];
    const float2 slF = mul2(sl, S.tab[cq][j]), slB = mul2(sl, S.tab[kCPW - 1 - cq][j]);
    const float2 kf = S.tab[q][j];                              // a^(KL q): CTA start -> chunk
    const float2 kb = S.tab[max(0, p.Tc / KL - 1 - q)][j];      // chunk end -> CTA end
    // carries into the chunk: from the left at its start, from the right at its end
    const float2 As = fma2(slw, lo2(X), fma2(slF, lo2(XW), mul2(kf, cs_af)));
    const float2 Cs = fma2(slw, hi2(X), fma2(slF, hi2(XW), mul2(kf, cs_cf)));
    const float2 Be = fma2(slw, lo2(Y), fma2(slB, lo2(YW), mul2(kb, cs_bb)));
    const float2 De = fma2(slw, hi2(Y), fma2(slB, hi2(YW), mul2(kb, cs_db)));

    float2 pw[kL];
    pw[0] = f2(1.0f);
#pragma unroll
    for (int i = 1; i < kL; ++i) pw[i] = min2(mul2(pw[i - 1], alpha), f2(0x1p126f));
    // results go to the first input tile (dead since the load phase), at the
    // same conflict-free offsets, then leave as coalesced 16-byte stores
    char* tout = smem;
    // carries into sub-chunk 1 from the left and into sub-chunk 0 from the
    // right: the other sub-chunk's total joins them (16-token chunks)
    const float2 A1 = fma2(slw, lo2(F0s), mul2(a8, As)), C1 = fma2(slw, hi2(F0s), mul2(a8, Cs));
    const float2 B0 = fma2(slw, lo2(G1s), mul2(a8, Be)), D0 = fma2(slw, hi2(G1s), mul2(a8, De));
#pragma unroll
    for (int st = 0; st < kH; ++st) {
        const int h = st ^ rot;
        float2 Ah = As, Ch = Cs, Bh = Be, Dh = De;
        if (kH == 2) {
            const bool first = h == 0;
            Ah = first ? As : A1;
            Ch = first ? Cs : C1;
            Bh = first ? B0 : Be;
            Dh = first ? D0 : De;
        }
        const float2 sh = mul2(slw, eh[st]);
        const int rowoff = (q * kH + h) * RB + j * PB;
#pragma unroll
        for (int i = 0; i < kL; ++i) {
            const float2 num = fma2(sh, n[st][i], fma2(pw[i], Ah, mul2(pw[kL - 1 - i], Bh)));
            float2 den = fma2(sh, dd[st][i], fma2(pw[i], Ch, mul2(pw[kL - 1 - i], Dh)));
            if (GATE) {
                // read before the result overwrites the first slot
                const int o = rowoff + i * SUB;
                const float2 g = make_float2(lds_f32(smem + SR * (QS ? 2 : 1) * p.tile_bytes + o),
                                             lds_f32(smem + G1 * p.tile_bytes + o));
                den = fma2(den, g, den);
            }
            Io<IO>::st_pair(tout + rowoff + i * SUB, mul2(num, rcp(den)));
        }
    }
    if (p.tma_store) {
        // lane i of warp 0 stores sub-tile i: boxes of 256 strided tokens,
        // clipped at T by the tensor map
        fence_proxy_async_smem();
        __syncthreads();
        if (tid < kL) {
            const int nbox = (tend - t0 + 255) / 256;
            for (int hb = 0; hb < nbox; ++hb)
                tma_store_3d(&p.omap, tout + tid * SUB + hb * 32 * RB, c0, t0 + tid + 256 * hb, b);
            bulk_commit_and_wait_read();
        }
    } else {
        __syncthreads();
        constexpr int UPS = SUB / 16;  // 16-byte units per sub-tile
        char* gout = p.out + ((size_t)b * p.T + t0) * p.C * es + (size_t)c0 * es;
#pragma unroll
        for (int u = tid; u < kL * UPS; u += kThreads) {
            const int i = u / UPS, o = (u - i * UPS) * 16;
            const int t = (o / RB) * kL + i;  // token within the CTA
            if (t0 + t < tend)
                *reinterpret_cast<uint4*>(gout + (size_t)t * p.C * es + (o % RB)) =
                    *reinterpret_cast<const uint4*>(tout + i * SUB + o);
        }
    }
    // no closing cluster barrier: every peer's store into this CTA's mailbox
    // completed before its mailbox wait, and nobody touches another CTA's
    // memory after that
    if (GX) {
        // count the CTA out; the last one resets the counters for the next
        // launch and advances the generation
        if (tid == 0) {
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
}

}  // namespace fast
}  // namespace vrwkv
