// Dense projections of the spatial-mix block ("Vision-RWKV Backbone",
// Overall Architecture, eq. 1-2: R, K, V = Q-Shift(X) W_R, W_K, W_V and the
// output projection W_O) on the 5th-generation tensor cores, sm_100a:
//
//   D[M, N] = A[M, K] * Bt[N, K]^T     A, Bt, D row-major bfloat16,
//                                      float32 accumulation in tensor memory.
//
// Persistent kernel, one CTA per SM, 192 threads in three roles:
//  * warp 0, one lane: TMA producer.  A (128 x 64) and Bt (256 x 64) tiles
//    arrive with the 128-byte swizzle into a ring of 4 shared-memory stages,
//    completing on the stage's "full" mbarrier.
//  * warp 1: allocates 512 tensor-memory columns (two 128 x 256 float32
//    accumulators); one lane issues tcgen05.mma kind::f16 (K = 16 per
//    instruction, four per stage) and frees each stage with tcgen05.commit
//    onto its "empty" mbarrier; after a tile's last stage it commits onto
//    the accumulator's "full" barrier.
//  * warps 2-5: epilogue.  Warp w reads tensor-memory lanes 32 (w mod 4) ..
//    +31 (rows of the tile) with tcgen05.ld, 32 columns at a time, converts
//    to bfloat16 and stores the rows; then releases the accumulator, so the
//    MMAs of the next tile overlap this epilogue.
// Output tiles are taken round-robin, N fastest, so the CTAs working at one
// time share A rows in L2 (Bt, the weights, stays resident in L2).
// Every mbarrier wait is bounded (the library's wait limit): a wait that runs
// out records flag 8 in the device error word, makes every role leave its
// loop, waits (bounded) for the copies and MMAs already issued and frees the
// tensor memory before the CTA exits.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "biwkv_tma.cuh"

namespace vrwkv {
namespace tcgemm {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kStages = 4;
constexpr int kAcc = 2;                       // accumulator buffers in tensor memory
constexpr int kTmemCols = kAcc * BN;          // 512: all of an SM's tensor memory
constexpr int kThreads = 192;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr unsigned kErrFlag = 8u;

struct Params {
    CUtensorMap ma;  // A as (K, M): box (64, 128), 128-byte swizzle
    CUtensorMap mb;  // Bt as (K, N): box (64, 256), 128-byte swizzle
    __nv_bfloat16* d;
    int M, N, K;
    unsigned int* err;
};

// Epilogue staging of one warp: 32 rows x 32 bfloat16 columns, 64 bytes a
// row; 16-byte piece c of row r sits at piece c ^ ((r >> 1) & 3), which keeps
// the row-wise writes and the piece-wise reads free of bank conflicts.
constexpr int kStgRowWords = 16;
__device__ __forceinline__ int stg_piece(int r, int c) { return c ^ ((r >> 1) & 3); }

// One warp's 32 x 32 chunk of results (lane = row row0 + lane, 32 float32
// columns from col), rounded to bfloat16.  A whole chunk passes through the
// warp's staging buffer so each store instruction covers 64-byte segments of
// eight rows instead of 16-byte pieces of 32 rows; a ragged one is stored
// row by row.
__device__ __forceinline__ void store_chunk(const uint32_t (&v)[32], uint32_t* stg, int lane, int row0, int col,
                                            int M, int N, __nv_bfloat16* d) {
    const int row = row0 + lane;
    if (row0 + 32 <= M && col + 32 <= N && (N % 8) == 0) {  // warp-uniform
        uint32_t* mine = stg + lane * kStgRowWords;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint32_t w4[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 h =
                    __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]), __uint_as_float(v[8 * q + 2 * e + 1]));
                w4[e] = *reinterpret_cast<const uint32_t*>(&h);
            }
            *reinterpret_cast<uint4*>(mine + 4 * stg_piece(lane, q)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // lane l: row 8 i + l / 4, 16-byte piece l % 4
            const int r = 8 * i + (lane >> 2), pc = lane & 3;
            const uint4 w = *reinterpret_cast<const uint4*>(stg + r * kStgRowWords + 4 * stg_piece(r, pc));
            *reinterpret_cast<uint4*>(d + (size_t)(row0 + r) * N + col + 8 * pc) = w;
        }
        __syncwarp();
    } else if (row < M && col < N) {
        uint32_t w16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            w16[e] = *reinterpret_cast<const uint32_t*>(&h);
        }
        __nv_bfloat16* dst = d + (size_t)row * N + col;
        if (col + 32 <= N && (N % 8) == 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int q = 0; q < 4; ++q) d4[q] = make_uint4(w16[4 * q], w16[4 * q + 1], w16[4 * q + 2], w16[4 * q + 3]);
        } else {
            for (int e = 0; e < 32 && col + e < N; ++e) {
                const uint32_t wv = w16[e >> 1];
                const unsigned short hv = (e & 1) ? (unsigned short)(wv >> 16) : (unsigned short)(wv & 0xffffu);
                dst[e] = __ushort_as_bfloat16(hv);
            }
        }
    }
}

struct alignas(1024) Smem {
    uint8_t a[kStages][A_BYTES];
    uint8_t b[kStages][B_BYTES];
    uint32_t stg[4][32 * kStgRowWords];  // epilogue staging, per epilogue warp
    unsigned long long full[kStages], empty[kStages];
    unsigned long long tfull[kAcc], tempty[kAcc];
    unsigned long long drain;  // completion of every issued MMA (abort path)
    unsigned tmem_base;
    int abort;
};

// Shared-memory matrix descriptor of a K-major tile with the 128-byte
// swizzle: 8-row groups 1024 bytes apart (stride byte offset 64 x 16 B),
// leading byte offset 1 (unused by the swizzled K-major layout), descriptor
// version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)64 << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: float32 accumulator, bfloat16 A and
// B, both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1,
                                            unsigned long long* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(fast::smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(fast::smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_test(unsigned long long* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(fast::smem_u32(bar)), "r"(parity), "r"(100000u)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase of parity `parity`; false if it ran out or the
// CTA is aborting (the first to run out records the failure).
__device__ __forceinline__ bool wait_phase(unsigned long long* bar, unsigned parity, volatile int* abort,
                                           unsigned* err) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
    while (!mbar_test(bar, parity)) {
        if (*abort) return false;
        if (fast::global_ns() - t0 > lim) {
            atomicOr(err, kErrFlag);
            *abort = 1;
            return false;
        }
    }
    return true;
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(fast::smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(unsigned long long* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     fast::smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 consecutive float32 columns of one tensor-memory lane per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    // load and wait in one statement: no use of v can be scheduled between
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
          "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
          "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
          "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr)
        : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) char smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (fast::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = (p.N + BN - 1) / BN, mt = (p.M + BM - 1) / BM;
    const int ntiles = nt * mt, nk = (p.K + BK - 1) / BK;
    volatile int* abort = &S.abort;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            fast::mbar_init(&S.full[s], 1);
            fast::mbar_init(&S.empty[s], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            fast::mbar_init(&S.tfull[a], 1);
            fast::mbar_init(&S.tempty[a], 4);  // one arrival per epilogue warp
        }
        fast::mbar_init(&S.drain, 1);
        S.abort = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         fast::smem_u32(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // producer: one A and one Bt tile per stage
            int it = 0;
            int last_par[kStages];
            for (int s = 0; s < kStages; ++s) last_par[s] = -1;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
                const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase(&S.empty[s], ph ^ 1u, abort, p.err)) break;
                    fast::mbar_expect_tx(&S.full[s], STAGE_BYTES);
                    tma_load_2d(S.a[s], &p.ma, kb * BK, m0, &S.full[s]);
                    tma_load_2d(S.b[s], &p.mb, kb * BK, n0, &S.full[s]);
                    last_par[s] = (int)ph;
                }
            }
            if (*abort) {
                // let the copies already issued land before the CTA exits
                for (int s = 0; s < kStages; ++s) {
                    if (last_par[s] < 0) continue;
                    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                    while (!mbar_test(&S.full[s], (unsigned)last_par[s]) && fast::global_ns() - t0 <= lim) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // MMA issuer
            int it = 0, lt = 0;
            bool issued = false;
            for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++lt) {
                const int acc = lt & 1;
                const unsigned aph = (lt >> 1) & 1;
                if (!wait_phase(&S.tempty[acc], aph ^ 1u, abort, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase(&S.full[s], ph, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(fast::smem_u32(S.a[s]));
                    const uint64_t bd = sw128_desc(fast::smem_u32(S.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)  // 32 bytes of K per instruction
                        tc_mma(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), kIdesc,
                               (kb > 0 || k > 0) ? 1u : 0u);
                    issued = true;
                    tc_commit(&S.empty[s]);
                }
                if (!ok) break;
                tc_commit(&S.tfull[acc]);
            }
            if (*abort && issued) {
                // every MMA issued so far completes before the memory is freed
                tc_commit(&S.drain);
                const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                while (!mbar_test(&S.drain, 0) && fast::global_ns() - t0 <= lim) {
                }
            }
        }
    } else {
        // epilogue: warp w reads tensor-memory lanes 32 (w mod 4) .. + 31
        const int quad = warp & 3;
        int lt = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++lt) {
            const int acc = lt & 1;
            const unsigned aph = (lt >> 1) & 1;
            if (!wait_phase(&S.tfull[acc], aph, abort, p.err)) break;
            tc_fence_after();
            const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
            const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)(c * 32), v);
                store_chunk(v, S.stg[warp - 2], lane, m0 + quad * 32, n0 + c * 32, p.M, p.N, p.d);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tempty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

// ---------------------------------------------------------------------------
// The same product on CTA pairs (cta_group::2): a cluster of two CTAs on two
// SMs computes a 256 x 256 output tile.  CTA r of the pair loads rows
// 128 r .. of the A tile and rows 128 r .. of the Bt tile (128 x 64 each,
// 32 KB per stage instead of 48: a 6-stage ring fits), and both copies
// complete on the leader's "full" barrier; the leader issues tcgen05.mma
// cta_group::2 (M = 256, N = 256, K = 16), which reads A and B from both
// CTAs' shared memory and accumulates each CTA's 128 rows in its own tensor
// memory; tcgen05.commit with a CTA mask frees the stage (and later hands
// the accumulator to the epilogue) in both CTAs.  No load is multicast:
// each CTA fetches only its own halves.
// ---------------------------------------------------------------------------
namespace pair {

constexpr int BM = 256, BN = 256, BK = 64;   // per cluster
constexpr int kHalf = 128;                   // rows of A and of Bt per CTA
constexpr int kStages = 6;
constexpr int A_BYTES = kHalf * BK * 2;      // 16 KB
constexpr int B_BYTES = kHalf * BK * 2;      // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;

struct alignas(1024) Smem {
    uint8_t a[kStages][A_BYTES];
    uint8_t b[kStages][B_BYTES];
    uint32_t stg[4][32 * kStgRowWords];  // epilogue staging, per epilogue warp
    unsigned long long full[kStages], empty[kStages];
    unsigned long long tfull[kAcc], tempty[kAcc];
    unsigned long long drain;
    unsigned tmem_base;
    int abort;
};

// kind::f16, float32 accumulator, bfloat16 A and B, both K-major, N = 256,
// M = 256 (the pair).
constexpr uint32_t kIdesc2 = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                             ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA load into this CTA's shared memory that completes on the leader's
// barrier (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map, int c0, int c1,
                                                 uint32_t leader_bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(fast::smem_u32(dst)),
        "l"(reinterpret_cast<unsigned long long>(map)), "r"(c0), "r"(c1), "r"(leader_bar)
        : "memory");
}
__device__ __forceinline__ void commit_pair(unsigned long long* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            fast::smem_u32(bar)),
        "h"((unsigned short)0x3)
        : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc2), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_tc2_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) char smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (fast::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int nt = (p.N + BN - 1) / BN, mt = (p.M + BM - 1) / BM;
    const int ntiles = nt * mt, nk = (p.K + BK - 1) / BK;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    volatile int* abort = &S.abort;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            fast::mbar_init(&S.full[s], 1);
            fast::mbar_init(&S.empty[s], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            fast::mbar_init(&S.tfull[a], 1);
            fast::mbar_init(&S.tempty[a], 8);  // the epilogue warps of both CTAs
        }
        fast::mbar_init(&S.drain, 1);
        S.abort = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         fast::smem_u32(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any remote signal
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // producer: this CTA's halves of A and Bt, completing on the leader's barrier
            int it = 0;
            int last_par[kStages];
            for (int s = 0; s < kStages; ++s) last_par[s] = -1;
            for (int t = cid; t < ntiles && !*abort; t += ncl) {
                const int m0 = (t / nt) * BM + (int)rank * kHalf, n0 = (t % nt) * BN + (int)rank * kHalf;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase(&S.empty[s], ph ^ 1u, abort, p.err)) break;
                    const uint32_t lbar = fast::mapa_u32(fast::smem_u32(&S.full[s]), 0);
                    if (leader) fast::mbar_expect_tx(&S.full[s], 2 * STAGE_BYTES);
                    tma_load_2d_pair(S.a[s], &p.ma, kb * BK, m0, lbar);
                    tma_load_2d_pair(S.b[s], &p.mb, kb * BK, n0, lbar);
                    last_par[s] = (int)ph;
                }
            }
            if (*abort && leader) {
                for (int s = 0; s < kStages; ++s) {
                    if (last_par[s] < 0) continue;
                    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                    while (!mbar_test(&S.full[s], (unsigned)last_par[s]) && fast::global_ns() - t0 <= lim) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // MMA issuer (the pair's leader)
            int it = 0, lt = 0;
            bool issued = false;
            for (int t = cid; t < ntiles && !*abort; t += ncl, ++lt) {
                const int acc = lt & 1;
                const unsigned aph = (lt >> 1) & 1;
                if (!wait_phase(&S.tempty[acc], aph ^ 1u, abort, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase(&S.full[s], ph, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(fast::smem_u32(S.a[s]));
                    const uint64_t bd = sw128_desc(fast::smem_u32(S.b[s]));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_pair(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k), (kb > 0 || k > 0) ? 1u : 0u);
                    issued = true;
                    commit_pair(&S.empty[s]);
                }
                if (!ok) break;
                commit_pair(&S.tfull[acc]);
            }
            if (*abort && issued) {
                tc_commit(&S.drain);
                const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                while (!mbar_test(&S.drain, 0) && fast::global_ns() - t0 <= lim) {
                }
            }
        }
    } else {
        // epilogue: this CTA's 128 rows of the pair's tile, 32 x 32 chunks per
        // warp through its staging buffer
        const int quad = warp & 3;
        const uint32_t leader_tempty[2] = {fast::mapa_u32(fast::smem_u32(&S.tempty[0]), 0),
                                           fast::mapa_u32(fast::smem_u32(&S.tempty[1]), 0)};
        int lt = 0;
        for (int t = cid; t < ntiles; t += ncl, ++lt) {
            const int acc = lt & 1;
            const unsigned aph = (lt >> 1) & 1;
            if (!wait_phase(&S.tfull[acc], aph, abort, p.err)) break;
            tc_fence_after();
            const int m0 = (t / nt) * BM, n0 = (t % nt) * BN;
            const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)(c * 32), v);
                store_chunk(v, S.stg[warp - 2], lane, m0 + (int)rank * kHalf + quad * 32, n0 + c * 32, p.M, p.N,
                            p.d);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_remote(leader_tempty[acc]);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while its pair may still signal it
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

}  // namespace pair

// ---------------------------------------------------------------------------
// The three token projections of the spatial-mix block with the Q-Shift mix
// as the A operand's producer ("Vision-RWKV Backbone", Overall Architecture,
// eq. 1: R, K, V = (mu x + (1 - mu) x-dagger) W, x-dagger per
// Quad-Directional Token Shift, eq. 9).  Same CTA-pair tiles and pipeline as
// gemm_tc2_kernel, plus:
//  * per stage, x and its Q-Shifted copy arrive by TMA from x's image view
//    (C, W, H, B): the shifted box is the same box displaced by +-s along w
//    or h, and TMA's zero fill is Q-Shift's border; a 64-channel K block lies
//    in one channel group, so one displacement serves the whole box;
//  * four groups of four mix warps, one per stage, turn x into the mix in
//    place, each thread one 128-byte row (the 128-byte swizzle permutes
//    16-byte chunks within a row, and the mix is element-wise, so chunk c of
//    a row pairs with chunk c of the shifted row and with mu of its logical
//    channels), with the
//    rounding of the stand-alone mix kernel (mu x and (1 - mu) x-dagger, each
//    rounded, then their sum): the A operand is the staged mix bit for bit;
//  * the leader's "full" barrier waits for both CTAs' mixes as well as the
//    B bytes; tiles run M block by M block over the three projections, so
//    the x tiles of one M block are read from HBM once.
// The mixed tokens never go to HBM.
// ---------------------------------------------------------------------------
namespace qsmix {

using pair::BM;
using pair::BN;
using pair::BK;
using pair::kHalf;
constexpr int kStages = 4;
constexpr int A_BYTES = kHalf * BK * 2;  // 16 KB: 128 rows x 64 channels
constexpr int B_BYTES = kHalf * BK * 2;
constexpr int kMixGroups = kStages;          // mix group g owns stage g (stages in flight: all)
constexpr int kMixGroupThreads = 128;        // one thread per row of a CTA's A tile
constexpr int kThreadsQ = 192 + kMixGroups * kMixGroupThreads;  // producer, MMA, 4 epilogue, 16 mix warps
constexpr int kMaxC = 1024;                  // mu of three projections in shared memory

struct Params {
    CUtensorMap mx;     // x as (C, W, H, B): box (64, bw, bh, 1) = 128 tokens, 128-byte swizzle
    CUtensorMap mb[3];  // Wt of each projection as (K, N): box (64, 128), 128-byte swizzle
    const float* mu[3];
    __nv_bfloat16* d[3];
    int M, N, K;        // M = B T tokens, N = K = C
    int T, W;
    int s;              // shift
    QsBounds g;
    int ng;             // shifted groups (4, or 2 for the bidirectional shift)
    int nproj;
    unsigned int* err;
};

struct alignas(1024) Smem {
    uint8_t a[kStages][A_BYTES];   // x, then the mix in place: the MMA's A operand
    uint8_t b[kStages][B_BYTES];
    uint8_t xs[kStages][A_BYTES];  // the Q-Shifted x
    float mu[3][kMaxC];
    float om[3][kMaxC];  // 1 - mu, rounded once
    uint32_t stg[4][32 * kStgRowWords];  // epilogue staging, per epilogue warp
    unsigned long long full[kStages], empty[kStages], xfull[kStages];
    unsigned long long tfull[kAcc], tempty[kAcc];
    unsigned long long drain;
    unsigned tmem_base;
    int abort;
    int mixok[kMixGroups];  // each mix group's verdict on its current stage
};

// The channel group's displacement (dw, dh) of a K block; 4: copied.
__device__ __forceinline__ int k_group(int k0, const Params& p) {
    int grp = qs_group(k0, p.g);
    return grp >= p.ng ? 4 : grp;
}

__device__ __forceinline__ bool mbar_test_cluster(unsigned long long* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(fast::smem_u32(bar)), "r"(parity), "r"(100000u)
        : "memory");
    return ok != 0;
}
// Bounded cluster-scope wait (the leader's full barrier takes the other
// CTA's release arrivals).
__device__ __forceinline__ bool wait_phase_cluster(unsigned long long* bar, unsigned parity, volatile int* abort,
                                                   unsigned* err) {
    if (mbar_test_cluster(bar, parity)) return true;
    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
    while (!mbar_test_cluster(bar, parity)) {
        if (*abort) return false;
        if (fast::global_ns() - t0 > lim) {
            atomicOr(err, kErrFlag);
            *abort = 1;
            return false;
        }
    }
    return true;
}
// named barrier 1 + g of mix group g
__device__ __forceinline__ void group_sync(int g) {
    asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(kMixGroupThreads) : "memory");
}

// (M block, projection, N block) of tile t: the projections of one M block
// are consecutive, so concurrent clusters share its x tiles through L2.
struct Tile {
    int mb, proj, nb;
};
__device__ __forceinline__ Tile tile_of(int t, int nt, int nproj) {
    Tile r;
    r.mb = t / (nt * nproj);
    const int rem = t - r.mb * nt * nproj;
    r.proj = rem / nt;
    r.nb = rem - r.proj * nt;
    return r;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreadsQ, 1)
    gemm_qs2_kernel(const __grid_constant__ Params p) {
    extern __shared__ __align__(1024) char smem_raw[];
    Smem& S = *reinterpret_cast<Smem*>(smem_raw + ((1024u - (fast::smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = pair::cluster_rank();
    const bool leader = rank == 0;
    const int nt = (p.N + BN - 1) / BN, mt = (p.M + BM - 1) / BM;
    const int ntiles = nt * mt * p.nproj, nk = (p.K + BK - 1) / BK;
    const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
    volatile int* abort = &S.abort;

    for (int e = tid; e < p.nproj * p.K; e += kThreadsQ) {
        const int pj = e / p.K, c = e - pj * p.K;
        const float m = __ldg(p.mu[pj] + c);
        S.mu[pj][c] = m;
        S.om[pj][c] = __fsub_rn(1.0f, m);
    }
    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) {
            // the leader's full barrier: its producer's expect_tx and both mixes
            fast::mbar_init(&S.full[st], 3);
            fast::mbar_init(&S.empty[st], 1);
            fast::mbar_init(&S.xfull[st], 1);
        }
        for (int a = 0; a < kAcc; ++a) {
            fast::mbar_init(&S.tfull[a], 1);
            fast::mbar_init(&S.tempty[a], 8);  // the epilogue warps of both CTAs
        }
        fast::mbar_init(&S.drain, 1);
        S.abort = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         fast::smem_u32(&S.tmem_base)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    pair::cluster_sync_all();  // both CTAs' barriers exist before any remote signal
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        if (lane == 0) {
            // producer: x and its shift into this CTA's stage (local barrier),
            // this CTA's half of Bt (the leader's barrier)
            int it = 0;
            int last_par[kStages];
            for (int st = 0; st < kStages; ++st) last_par[st] = -1;
            for (int t = cid; t < ntiles && !*abort; t += ncl) {
                const Tile tl = tile_of(t, nt, p.nproj);
                const int m_cta = tl.mb * BM + (int)rank * kHalf;  // this CTA's first token
                const int bidx = m_cta / p.T, tok = m_cta - bidx * p.T;
                const int hrow = tok / p.W, w0 = tok - hrow * p.W;
                const int n0 = tl.nb * BN + (int)rank * kHalf;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int st = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase(&S.empty[st], ph ^ 1u, abort, p.err)) break;
                    const int k0 = kb * BK;
                    const int grp = k_group(k0, p);
                    const uint32_t lbar = fast::mapa_u32(fast::smem_u32(&S.full[st]), 0);
                    if (leader) fast::mbar_expect_tx(&S.full[st], 2 * B_BYTES);
                    fast::mbar_expect_tx(&S.xfull[st], (unsigned)(grp < 4 ? 2 * A_BYTES : A_BYTES));
                    fast::tma_load_4d(S.a[st], &p.mx, k0, w0, hrow, bidx, &S.xfull[st]);
                    if (grp < 4) {
                        const int dw = grp == 0 ? -p.s : (grp == 1 ? p.s : 0);
                        const int dh = grp == 2 ? -p.s : (grp == 3 ? p.s : 0);
                        fast::tma_load_4d(S.xs[st], &p.mx, k0, w0 + dw, hrow + dh, bidx, &S.xfull[st]);
                    }
                    pair::tma_load_2d_pair(S.b[st], &p.mb[tl.proj], k0, n0, lbar);
                    last_par[st] = (int)ph;
                }
            }
            if (*abort) {
                // let this CTA's copies land before it leaves
                for (int st = 0; st < kStages; ++st) {
                    if (last_par[st] < 0) continue;
                    const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                    while (!mbar_test(&S.xfull[st], (unsigned)last_par[st]) && fast::global_ns() - t0 <= lim) {
                    }
                    if (leader)
                        while (!mbar_test_cluster(&S.full[st], (unsigned)last_par[st]) &&
                               fast::global_ns() - t0 <= lim) {
                        }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // MMA issuer (the pair's leader)
            int it = 0, lt = 0;
            bool issued = false;
            for (int t = cid; t < ntiles && !*abort; t += ncl, ++lt) {
                const int acc = lt & 1;
                const unsigned aph = (lt >> 1) & 1;
                if (!wait_phase(&S.tempty[acc], aph ^ 1u, abort, p.err)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
                bool ok = true;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int st = it % kStages;
                    const unsigned ph = (it / kStages) & 1;
                    if (!wait_phase_cluster(&S.full[st], ph, abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = sw128_desc(fast::smem_u32(S.a[st]));
                    const uint64_t bd = sw128_desc(fast::smem_u32(S.b[st]));
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        pair::mma_pair(d_tmem, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k),
                                       (kb > 0 || k > 0) ? 1u : 0u);
                    issued = true;
                    pair::commit_pair(&S.empty[st]);
                }
                if (!ok) break;
                pair::commit_pair(&S.tfull[acc]);
            }
            if (*abort && issued) {
                tc_commit(&S.drain);
                const unsigned long long t0 = fast::global_ns(), lim = fast::g_vrwkv_wait_ns;
                while (!mbar_test(&S.drain, 0) && fast::global_ns() - t0 <= lim) {
                }
            }
        }
    } else if (warp < 6) {
        // epilogue: this CTA's 128 rows of the pair's tile
        const int quad = warp & 3;
        const uint32_t leader_tempty[2] = {fast::mapa_u32(fast::smem_u32(&S.tempty[0]), 0),
                                           fast::mapa_u32(fast::smem_u32(&S.tempty[1]), 0)};
        int lt = 0;
        for (int t = cid; t < ntiles; t += ncl, ++lt) {
            const int acc = lt & 1;
            const unsigned aph = (lt >> 1) & 1;
            if (!wait_phase(&S.tfull[acc], aph, abort, p.err)) break;
            tc_fence_after();
            const Tile tl = tile_of(t, nt, p.nproj);
            const int m0 = tl.mb * BM, n0 = tl.nb * BN;
            const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tbase + (uint32_t)(c * 32), v);
                store_chunk(v, S.stg[warp - 2], lane, m0 + (int)rank * kHalf + quad * 32, n0 + c * 32, p.M, p.N,
                            p.d[tl.proj]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) pair::arrive_remote(leader_tempty[acc]);
        }
    } else {
        // mix warps: group g (four warps) mixes every stage-g tile; thread r of
        // the group owns row r of this CTA's 128-row A tile.  The groups work
        // on their stages concurrently, so a stage's mix latency overlaps the
        // MMAs of the others.
        const int gi = (warp - 6) >> 2;
        const int r = tid - 192 - gi * kMixGroupThreads;
        const uint32_t rowoff = (uint32_t)r * 128u;
        int it = 0;
        bool go = true;
        for (int t = cid; t < ntiles && go; t += ncl) {
            const Tile tl = tile_of(t, nt, p.nproj);
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int st = it % kStages;
                if (st != gi) continue;
                const unsigned ph = (it / kStages) & 1;
                if (r == 0) S.mixok[gi] = wait_phase(&S.xfull[st], ph, abort, p.err) ? 1 : 0;
                group_sync(gi);
                if (!S.mixok[gi]) {
                    go = false;
                    break;
                }
                const int k0 = kb * BK;
                const bool shifted = k_group(k0, p) < 4;
                const uint8_t* xa = S.a[st] + rowoff;
                const uint8_t* xd = (shifted ? S.xs[st] : S.a[st]) + rowoff;
                const float* mu = &S.mu[tl.proj][k0];
                const float* om = &S.om[tl.proj][k0];
#pragma unroll 4
                for (int c = 0; c < BK / 8; ++c) {
                    const uint32_t off = (uint32_t)((c ^ (r & 7)) * 16);  // chunk c's place in the swizzled row
                    const uint4 xv = *reinterpret_cast<const uint4*>(xa + off);
                    const uint4 dv = *reinterpret_cast<const uint4*>(xd + off);
                    const float4 m0 = *reinterpret_cast<const float4*>(mu + 8 * c);
                    const float4 m1 = *reinterpret_cast<const float4*>(mu + 8 * c + 4);
                    const float4 o0 = *reinterpret_cast<const float4*>(om + 8 * c);
                    const float4 o1 = *reinterpret_cast<const float4*>(om + 8 * c + 4);
                    const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
                    const float ov[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
                    const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w}, dw[4] = {dv.x, dv.y, dv.z, dv.w};
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // mu x + (1 - mu) x-dagger, each operation rounded on its own
                        // (no contraction into a multiply-add)
                        const float lo = __fadd_rn(__fmul_rn(mv[2 * e], __uint_as_float(xw[e] << 16)),
                                                   __fmul_rn(ov[2 * e], __uint_as_float(dw[e] << 16)));
                        const float hi = __fadd_rn(__fmul_rn(mv[2 * e + 1], __uint_as_float(xw[e] & 0xffff0000u)),
                                                   __fmul_rn(ov[2 * e + 1], __uint_as_float(dw[e] & 0xffff0000u)));
                        const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
                        ow[e] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    *reinterpret_cast<uint4*>(const_cast<uint8_t*>(xa) + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                }
                // the mix is read by the tensor cores (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                group_sync(gi);
                if (r == 0) pair::arrive_remote(fast::mapa_u32(fast::smem_u32(&S.full[st]), 0));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    pair::cluster_sync_all();  // no CTA leaves while its pair may still signal it
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

}  // namespace qsmix

// W (K x N, row-major) -> Wt (N x K, row-major), 32 x 32 tiles through
// shared memory; the GEMM reads its B operand K-major.
template <typename T>
__global__ void __launch_bounds__(256) transpose_kernel(const T* __restrict__ w, T* __restrict__ wt, int K, int N) {
    __shared__ T tile[32][33];
    const int k0 = blockIdx.y * 32, n0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int k = k0 + r, n = n0 + tx;
        if (k < K && n < N) tile[r][tx] = w[(size_t)k * N + n];
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int n = n0 + r, k = k0 + tx;
        if (n < N && k < K) wt[(size_t)n * K + k] = tile[tx][r];
    }
}

// The same transpose for 16-bit elements two at a time: 64 x 64 tiles, each
// thread moving 4-byte pairs (rows of a warp access are 128 bytes instead of
// 64), the tile's rows padded to 33 words (at most 2-way bank conflicts when
// a warp reads a column of pairs).  Needs K and N even and every pointer
// 4-byte aligned.
// Up to four matrices in one launch: blockIdx.z picks the pair (w, wt).
template <typename T>
struct TransposeBatch {
    const T* w[4];
    T* wt[4];
};
template <typename T>
__global__ void __launch_bounds__(256) transpose2_kernel(const __grid_constant__ TransposeBatch<T> tb, int K, int N) {
    static_assert(sizeof(T) == 2, "16-bit elements");
    __shared__ uint32_t tile[64][33];  // [k][pair of n]
    const T* __restrict__ w = tb.w[blockIdx.z];
    T* __restrict__ wt = tb.wt[blockIdx.z];
    const int k0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int r = ty; r < 64; r += 8) {
        const int k = k0 + r, n = n0 + 2 * tx;
        tile[r][tx] = (k < K && n < N) ? *reinterpret_cast<const uint32_t*>(w + (size_t)k * N + n) : 0u;
    }
    __syncthreads();
    for (int c = ty; c < 64; c += 8) {
        const int n = n0 + c, k = k0 + 2 * tx;
        if (n < N && k < K) {
            const uint32_t a = tile[2 * tx][c >> 1], b = tile[2 * tx + 1][c >> 1];
            const uint32_t lo = (c & 1) ? (a >> 16) : (a & 0xffffu);
            const uint32_t hi = (c & 1) ? (b >> 16) : (b & 0xffffu);
            *reinterpret_cast<uint32_t*>(wt + (size_t)n * K + k) = lo | (hi << 16);
        }
    }
}

// float32 projections on the FP32 pipes (the bfloat16 path above is the
// tensor-core one): D = A W with W (K x N) row-major, 64 x 64 tiles, 4 x 4
// results per thread.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const float* __restrict__ a, const float* __restrict__ w,
                                                      float* __restrict__ d, int M, int N, int K) {
    __shared__ float As[16][64 + 4];
    __shared__ float Ws[16][64];
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int i = threadIdx.x; i < 16 * 64; i += 256) {
            const int kk = i & 15, mm = i >> 4;  // A tile, transposed into As[k][m]
            const int m = m0 + mm, k = k0 + kk;
            As[kk][mm] = (m < M && k < K) ? a[(size_t)m * K + k] : 0.f;
            const int nn = i & 63, kw = i >> 6;
            const int n = n0 + nn, kq = k0 + kw;
            Ws[kw][nn] = (n < N && kq < K) ? w[(size_t)kq * N + n] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float av[4], wv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) wv[j] = Ws[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], wv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n < N) d[(size_t)m * N + n] = acc[i][j];
        }
    }
}

}  // namespace tcgemm
}  // namespace vrwkv
