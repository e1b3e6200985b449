// C ABI of the Vision-RWKV spatial-mix core (declared in include/vrwkv.h):
// host-side argument validation, tiling decisions and kernel launches.
// Validation happens before any CUDA call, so invalid arguments are
// rejected without touching the device.
#include <algorithm>
#include <array>
#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>
#include <type_traits>
#include <utility>
#include <vector>

#include <cuda.h>

#include "vrwkv.h"
#include "biwkv.cuh"
#include "biwkv_tma.cuh"
#include "biwkv_tm.cuh"
#include "biwkv_wide.cuh"
#include "qshift.cuh"
#include "channel_mix.cuh"
#include "biwkv_bwd.cuh"
#include "biwkv_bwd_tm.cuh"
#include "layer_norm.cuh"
#include "gemm_tc.cuh"

// Device error word: set by kernels whose bounded waits ran out (bit 0).
__device__ unsigned int g_vrwkv_device_error;

namespace {

using namespace vrwkv;

thread_local std::string g_last_error;
thread_local const char* g_last_kernel = "";

vrwkv_status fail(vrwkv_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

vrwkv_status ok() {
    g_last_error.clear();
    return VRWKV_OK;
}

vrwkv_status cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(VRWKV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

int elem_bytes(vrwkv_dtype dt) { return dt == VRWKV_F32 ? 4 : 2; }

// Q-Shift channel-group bounds of the q_shift listing: int(C*gamma*j),
// j = 1..4, with C*gamma formed first and then multiplied by j, both in
// double precision (the listing's Python evaluation order), truncated.
QsBounds qs_bounds(int C, double gamma) {
    QsBounds g;
    const double cg = (double)C * gamma;
    for (int j = 0; j < 4; ++j) g.b[j] = (int)(cg * (double)(j + 1));
    return g;
}
QsBounds no_shift_bounds() { return QsBounds{{0, 0, 0, 0}}; }

// Every bound a multiple of n: vectors (or slabs) of n channels never
// straddle two groups.
bool bounds_multiple_of(const QsBounds& g, int n) {
    for (int j = 0; j < 4; ++j)
        if (g.b[j] % n != 0) return false;
    return true;
}

// Shifted channel groups of a Q-Shift mode: all four (eq. 9) or the two
// row groups (bidirectional shift of sparse inputs).
int shifted_groups(const vrwkv_qshift_params* qs) { return qs && qs->mode == VRWKV_QSHIFT_BIDIR ? 2 : 4; }


// Raise the dynamic shared-memory limit of a kernel once per size needed.
template <typename K>
cudaError_t ensure_smem(K kernel, std::atomic<int>& granted, int bytes) {
    if (bytes <= 48 * 1024 || bytes <= granted.load(std::memory_order_relaxed)) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) {
        int cur = granted.load();
        while (bytes > cur && !granted.compare_exchange_weak(cur, bytes)) {
        }
    }
    return e;
}

struct FusedPlan {
    FusedParams p;
    int ntiles;
    int layout;
    bool qs;
    dim3 grid;
    int threads;
    int smem;
};

template <typename IO, int LAYOUT, bool QS>
vrwkv_status launch_fused(const FusedPlan& pl, cudaStream_t stream) {
    static std::atomic<int> granted{0};
    auto kern = biwkv_fused_kernel<IO, LAYOUT, QS>;
    cudaError_t e = ensure_smem(kern, granted, pl.smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = pl.grid;
    cfg.blockDim = dim3(pl.threads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pl.p.ncl > 1 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, pl.p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_fused_kernel launch");
    g_last_kernel = "biwkv_fused_kernel";
    return ok();
}

template <typename IO>
vrwkv_status dispatch_layout(const FusedPlan& pl, cudaStream_t s) {
    switch (pl.layout * 2 + (pl.qs ? 1 : 0)) {
    case kKV * 2 + 0: return launch_fused<IO, kKV, false>(pl, s);
    case kKV * 2 + 1: return launch_fused<IO, kKV, true>(pl, s);
    case kRKV * 2 + 0: return launch_fused<IO, kRKV, false>(pl, s);
    case kRKV * 2 + 1: return launch_fused<IO, kRKV, true>(pl, s);
    case kX * 2 + 0: return launch_fused<IO, kX, false>(pl, s);
    default: return launch_fused<IO, kX, true>(pl, s);
    }
}

// ---------------------------------------------------------------------------
// TMA fast path
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// Device address of the error word on the current device (looked up once per
// device; the symbol's host-side name is not a device address).
unsigned int* device_error_word() {
    static unsigned int* addr[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_vrwkv_device_error) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned int*>(a);
    }
    return addr[dev];
}

// Fixed device workspace of vrwkv_spatial_gate_static, for callers that
// cannot allocate device memory: it is reserved when the module loads, so a
// call allocates nothing.  4 MiB holds the exchange state of about 1600
// (batch row, 8-channel slab) columns (2624 bytes each).  One array per device, shared by every
// caller of that entry point.
constexpr size_t kStaticWsBytes = 4u << 20;
static __device__ __align__(256) unsigned char g_vrwkv_static_ws[kStaticWsBytes];

// Address of the current device's static workspace (nullptr if unknown).
unsigned char* static_workspace() {
    static std::mutex mu;
    static unsigned char* addr[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* a = nullptr;
        if (cudaGetSymbolAddress(&a, g_vrwkv_static_ws) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned char*>(a);
    }
    return addr[dev];
}

// ---- dense projections (tcgen05 GEMM for bfloat16, FP32 pipes for float32) ----
// VRWKV_GEMM_1CTA=1 keeps the projections on single-CTA tiles (diagnostics).
bool gemm_single_cta_forced() {
    const char* e = getenv("VRWKV_GEMM_1CTA");
    return e && e[0] == '1';
}

int sm_count() {
    static int n[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!n[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        n[dev] = v;
    }
    return n[dev];
}

// D (M x N) = X (M x K) * W (K x N), all row-major.  bfloat16: W is first
// transposed into wt (N x K, the K-major B operand) and the product runs on
// the tensor cores with float32 accumulation; float32: on the FP32 pipes.
// n matrices W[i] (K x N, bfloat16, row-major) -> wt[i] (N x K) in one
// launch, two elements per thread access; false (nothing launched) unless
// the sizes are even and every pointer 4-byte aligned.
bool launch_transpose_pairs(const void* const* W, void* const* wt, int n, int K, int N, cudaStream_t s) {
    if (n < 1 || n > 4 || K % 2 != 0 || N % 2 != 0) return false;
    tcgemm::TransposeBatch<__nv_bfloat16> tb{};
    for (int i = 0; i < n; ++i) {
        if (!aligned(W[i], 4) || !aligned(wt[i], 4)) return false;
        tb.w[i] = static_cast<const __nv_bfloat16*>(W[i]);
        tb.wt[i] = static_cast<__nv_bfloat16*>(wt[i]);
    }
    const dim3 grid((unsigned)((N + 63) / 64), (unsigned)((K + 63) / 64), (unsigned)n);
    tcgemm::transpose2_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(tb, K, N);
    return true;
}

// W (K x N, bfloat16, row-major) -> wt (N x K): pairs of elements per thread
// where the sizes are even and the pointers 4-byte aligned, else one.
vrwkv_status launch_transpose(const void* W, void* wt, int K, int N, cudaStream_t s) {
    if (!launch_transpose_pairs(&W, &wt, 1, K, N, s)) {
        const dim3 grid((unsigned)((N + 31) / 32), (unsigned)((K + 31) / 32));
        tcgemm::transpose_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(W),
                                                                      static_cast<__nv_bfloat16*>(wt), K, N);
    }
    return cuda_status(cudaGetLastError(), "transpose launch");
}

vrwkv_status gemm_project(const void* X, const void* W, void* D, int M, int N, int K, vrwkv_dtype dtype,
                          void* wt, cudaStream_t s, bool wt_ready = false) {
    if (dtype == VRWKV_F32) {
        const dim3 grid((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64));
        tcgemm::gemm_f32_kernel<<<grid, 256, 0, s>>>(static_cast<const float*>(X), static_cast<const float*>(W),
                                                     static_cast<float*>(D), M, N, K);
        return cuda_status(cudaGetLastError(), "gemm_f32_kernel launch");
    }
    if (K % 8 != 0) return fail(VRWKV_ERR_UNSUPPORTED, "bfloat16 projections need C %% 8 == 0");
    if (!wt_ready) {  // else the caller transposed W into wt already
        vrwkv_status st = launch_transpose(W, wt, K, N, s);
        if (st != VRWKV_OK) return st;
    }
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(VRWKV_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    tcgemm::Params p;
    const cuuint32_t estr[2] = {1, 1};
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)tcgemm::BK, (cuuint32_t)tcgemm::BM};
        if (enc(&p.ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(VRWKV_ERR_UNSUPPORTED, "tensor map of the GEMM's A operand could not be encoded");
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)tcgemm::BK, (cuuint32_t)tcgemm::BN};
        if (enc(&p.mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wt, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return fail(VRWKV_ERR_UNSUPPORTED, "tensor map of the GEMM's B operand could not be encoded");
    }
    p.d = static_cast<__nv_bfloat16*>(D);
    p.M = M;
    p.N = N;
    p.K = K;
    p.err = device_error_word();
    if (!p.err) return fail(VRWKV_ERR_CUDA, "cannot locate the device error word");
    if (!gemm_single_cta_forced()) {
        // CTA pairs (cta_group::2): the B map's box holds one CTA's 128 rows
        tcgemm::Params p2 = p;
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)N};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)tcgemm::BK, (cuuint32_t)tcgemm::pair::kHalf};
        if (enc(&p2.mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wt, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS) {
            const int smem2 = (int)sizeof(tcgemm::pair::Smem) + 1024;
            static std::atomic<int> granted2{0};
            cudaError_t e2 = ensure_smem(tcgemm::pair::gemm_tc2_kernel, granted2, smem2);
            if (e2 == cudaSuccess) {
                const int tiles2 = ((M + tcgemm::pair::BM - 1) / tcgemm::pair::BM) *
                                   ((N + tcgemm::pair::BN - 1) / tcgemm::pair::BN);
                const int pairs = std::max(1, std::min(tiles2, sm_count() / 2));
                tcgemm::pair::gemm_tc2_kernel<<<2 * pairs, tcgemm::kThreads, smem2, s>>>(p2);
                e2 = cudaGetLastError();
                if (e2 == cudaSuccess) return ok();
            }
            cudaGetLastError();  // fall back to single CTAs
        }
    }
    const int smem = (int)sizeof(tcgemm::Smem) + 1024;
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem(tcgemm::gemm_tc_kernel, granted, smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    const int tiles = ((M + tcgemm::BM - 1) / tcgemm::BM) * ((N + tcgemm::BN - 1) / tcgemm::BN);
    const int grid = std::min(tiles, sm_count());
    tcgemm::gemm_tc_kernel<<<grid, tcgemm::kThreads, smem, s>>>(p);
    return cuda_status(cudaGetLastError(), "gemm_tc_kernel launch");
}

// VRWKV_BWD_TM=0 keeps the backward on the 8-token kernel (diagnostics and
// tests).
bool bwd_tm_disabled() {
    const char* e = getenv("VRWKV_BWD_TM");
    return e && e[0] == '0' && e[1] == 0;
}

// The 16-token tensor-memory backward (bwd2::biwkv_bwd_tm_kernel): sets
// *fell_back when the shape cannot be co-scheduled or more than four CTAs
// would share an SM.
// Cluster scheduling policy of the clustered kernels: spread by default
// (measured on the B200 with the tensor-memory forward at B=8, T=4096,
// C=1024: 83.0 us against 84.9 us with load balancing);
// VRWKV_CLUSTER_POLICY=l(oad balancing) or d(efault) for comparisons, and
// VRWKV_CLUSTER_POLICY_BWD / _NARROW for the backward and 8-channel kernels
// alone.
cudaClusterSchedulingPolicy cluster_policy(const char* var) {
    const char* e = getenv(var);
    if (!e || !e[0]) e = getenv("VRWKV_CLUSTER_POLICY");
    if (e && e[0] == 'l') return cudaClusterSchedulingPolicyLoadBalancing;
    if (e && e[0] == 'd') return cudaClusterSchedulingPolicyDefault;
    return cudaClusterSchedulingPolicySpread;
}

template <typename IO>
vrwkv_status launch_bwd_tm(const bwd::Params& p, cudaStream_t s, bool* fell_back) {
    auto kern = bwd2::biwkv_bwd_tm_kernel<IO>;
    const int smem = std::max((int)bwd2::Layout<IO>::kBytes, bwd2::kSmemFloor);
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem(kern, granted, smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.ncl, (p.C + bwd2::kCS - 1) / bwd2::kCS, p.B);
    cfg.blockDim = dim3(bwd2::kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cluster_policy("VRWKV_CLUSTER_POLICY_BWD");
    cfg.attrs = attr;
    cfg.numAttrs = p.ncl > 1 ? 2 : 0;
    static std::atomic<int> checked[bwd2::kClusterMax + 1];
    int v = checked[p.ncl].load();
    if (v == 0) {
        int per_sm = 0, nclu = 1;
        cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, bwd2::kThreads, smem);
        if (oe == cudaSuccess && p.ncl > 1) oe = cudaOccupancyMaxActiveClusters(&nclu, kern, &cfg);
        if (oe != cudaSuccess) cudaGetLastError();
        v = (oe == cudaSuccess && per_sm >= 1 && per_sm * bwd2::kTmemCols <= 512 && nclu > 0) ? 1 : -1;
        checked[p.ncl].store(v);
    }
    if (v < 0) {
        *fell_back = true;
        return VRWKV_OK;
    }
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_bwd_tm_kernel launch");
    g_last_kernel = "biwkv_bwd_tm_kernel";
    return ok();
}

// VRWKV_BLOCK_FUSED=1 projects R, K, V with the fused Q-Shift GEMM instead of
// staging the three mixes in HBM.  Off by default: measured on the B200 at
// B = 8, 64 x 64, C = 1024 the fused block takes 521 us against 424 us
// staged.  The fused A producer mixes every x tile once per N tile (four
// times per projection at C = 1024), and that element-wise work (about six
// instructions per element) outgrows what the SM issues beside the MMAs;
// staged, each element is mixed once per projection.
bool block_fused_wanted() {
    const char* e = getenv("VRWKV_BLOCK_FUSED");
    return e && e[0] == '1';
}

// R, K, V = mix_{r,k,v}(x) W_{r,k,v} in one launch of the fused Q-Shift GEMM
// (bfloat16).  Returns false (nothing launched) when the shape is outside its
// limits: C a multiple of 256 and at most 1024, 64-channel K blocks inside
// one channel group, 128-token tiles of whole image rows (or whole 128-token
// pieces of one row) inside one image, all three mu given.
bool gemm_qs_project(const void* x, const void* const* wts, const float* const* mus, void* const* dst,
                     int B, int T, int C, const vrwkv_qshift_params* qs, char* wt_slots, size_t wslot,
                     cudaStream_t s, vrwkv_status* st) {
    using namespace tcgemm::qsmix;
    if (!mus[0] || !mus[1] || !mus[2]) return false;
    if (C % 256 != 0 || C > kMaxC || T % 128 != 0) return false;
    const int W = qs->W, H = qs->H;
    if (!((W <= 128 && 128 % W == 0) || W % 128 == 0)) return false;
    const QsBounds g = qs_bounds(C, qs->gamma);
    if (!bounds_multiple_of(g, 64)) return false;
    if (!aligned(x, 16)) return false;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    Params p;
    {
        const int bw = W <= 128 ? W : 128, bh = W <= 128 ? 128 / W : 1;
        const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)B};
        const cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)T * C * 2};
        const cuuint32_t box[4] = {64u, (cuuint32_t)bw, (cuuint32_t)bh, 1u};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        if (enc(&p.mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    for (int i = 0; i < 3; ++i) {
        void* wt = wt_slots + i * wslot;
        {
            const vrwkv_status e = launch_transpose(wts[i], wt, C, C, s);
            if (e != VRWKV_OK) {
                *st = e;
                return true;
            }
        }
        const cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)C};
        const cuuint64_t strides[1] = {(cuuint64_t)C * 2};
        const cuuint32_t box[2] = {(cuuint32_t)tcgemm::BK, (cuuint32_t)tcgemm::pair::kHalf};
        const cuuint32_t estr[2] = {1, 1};
        if (enc(&p.mb[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, wt, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
            *st = fail(VRWKV_ERR_UNSUPPORTED, "tensor map of a projection's B operand could not be encoded");
            return true;
        }
        p.mu[i] = mus[i];
        p.d[i] = static_cast<__nv_bfloat16*>(dst[i]);
    }
    {
        vrwkv_status e0 = cuda_status(cudaGetLastError(), "transpose_kernel launch");
        if (e0 != VRWKV_OK) {
            *st = e0;
            return true;
        }
    }
    p.M = B * T;
    p.N = C;
    p.K = C;
    p.T = T;
    p.W = W;
    p.s = qs->shift_pixel;
    p.g = g;
    p.ng = shifted_groups(qs);
    p.nproj = 3;
    p.err = device_error_word();
    if (!p.err) {
        *st = fail(VRWKV_ERR_CUDA, "cannot locate the device error word");
        return true;
    }
    const int smem = (int)sizeof(Smem) + 1024;
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem(gemm_qs2_kernel, granted, smem);
    if (e != cudaSuccess) {
        *st = cuda_status(e, "cudaFuncSetAttribute");
        return true;
    }
    const int tiles = ((p.M + BM - 1) / BM) * (C / BN) * 3;
    const int pairs = std::max(1, std::min(tiles, sm_count() / 2));
    gemm_qs2_kernel<<<2 * pairs, kThreadsQ, smem, s>>>(p);
    *st = cuda_status(cudaGetLastError(), "gemm_qs2_kernel launch");
    return true;
}

// Workspace of vrwkv_spatial_mix_block: six (B, T, C) token buffers and the
// four transposed weight matrices, each 256-byte aligned.
size_t block_wt_slot(int C, vrwkv_dtype dtype) {
    return ((size_t)C * C * elem_bytes(dtype) + 255) / 256 * 256;
}
size_t block_ws_slot(int B, int T, int C, vrwkv_dtype dtype) {
    return ((size_t)B * T * C * elem_bytes(dtype) + 255) / 256 * 256;
}

// Launch shape of the column-walking kernels (channel mix, Q-Shift mixes):
// blocks of (tx vectors) x (ty rows), channel chunks of at most 256 vectors
// along x, and along y one wave of CTAs (SMs x resident CTAs per SM, from the
// occupancy of `kern`), each owning an equal share of the BT token rows.
template <typename K>
vrwkv_status column_launch(K kern, std::atomic<int>& occ, int UR, long long BT, dim3* grid, dim3* block) {
    const int nchunks = (UR + 255) / 256;
    int tx = (UR + nchunks - 1) / nchunks;
    if (nchunks > 1) tx = (tx + 31) / 32 * 32;
    const int ty = std::max(1, 256 / tx);
    int o = occ.load(std::memory_order_relaxed);
    if (o == 0) {
        int nb = 0;
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, tx * ty, 0);
        if (e != cudaSuccess) return cuda_status(e, "occupancy query");
        o = std::max(1, nb);
        occ.store(o, std::memory_order_relaxed);
    }
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long row_groups = (BT + ty * kCmRows - 1) / (ty * kCmRows);
    const long long gy = std::max<long long>(1, std::min<long long>(row_groups, (long long)sms * o / nchunks));
    *grid = dim3((unsigned)nchunks, (unsigned)gy);
    *block = dim3((unsigned)tx, (unsigned)ty);
    return VRWKV_OK;
}

// Q-Shift mixes of one x into NMIX outputs by the column walker; false when
// the vector conditions do not hold (the caller then takes another path).
template <int NMIX>
bool launch_qs_mix(const void* x, void* const* outs, const float* const* mus, int B, int H, int W, int C,
                   int shift, double gamma, int ng, vrwkv_dtype dtype, cudaStream_t s, vrwkv_status* st) {
    const int es = elem_bytes(dtype), nv = 16 / es;
    const long long BT = (long long)B * H * W;
    const QsBounds g = qs_bounds(C, gamma);
    if (C % nv != 0 || !bounds_multiple_of(g, nv) || BT > 0x7fffffffLL || !aligned(x, 16)) return false;
    for (int m = 0; m < NMIX; ++m)
        if (!aligned(outs[m], 16) || (mus[0] && !mus[m])) return false;
    QsMixParams<NMIX> q;
    ChannelMixParams& p = q.base;
    p.x = static_cast<const char*>(x);
    p.out = nullptr;
    p.mu_r = p.mu_k = nullptr;
    p.BT = (int)BT;
    p.T = H * W;
    p.C = C;
    p.H = H;
    p.W = W;
    p.s = shift;
    p.g = g;
    p.ng = ng;
    p.UR = C / nv;
    p.divT = make_fastdiv((unsigned)p.T);
    p.divW = make_fastdiv((unsigned)W);
    for (int m = 0; m < NMIX; ++m) {
        q.out[m] = static_cast<char*>(outs[m]);
        q.mu[m] = mus[0] ? mus[m] : nullptr;
    }
    static std::atomic<int> occ[2] = {{0}, {0}};
    dim3 grid, block;
    const int di = dtype == VRWKV_F32 ? 0 : 1;
    *st = dtype == VRWKV_F32 ? column_launch(qs_mix_vec_kernel<float, NMIX>, occ[di], p.UR, BT, &grid, &block)
                             : column_launch(qs_mix_vec_kernel<__nv_bfloat16, NMIX>, occ[di], p.UR, BT, &grid,
                                             &block);
    if (*st != VRWKV_OK) return true;
    if (dtype == VRWKV_F32) qs_mix_vec_kernel<float, NMIX><<<grid, block, 0, s>>>(q);
    else qs_mix_vec_kernel<__nv_bfloat16, NMIX><<<grid, block, 0, s>>>(q);
    *st = cuda_status(cudaGetLastError(), "qs_mix kernel launch");
    return true;
}

bool tma_disabled() {
    const char* e = getenv("VRWKV_DISABLE_TMA");
    return e && e[0] && e[0] != '0';
}

// VRWKV_NO_TMA_STORE=1 makes the forward TMA path write its results with
// plain 16-byte stores instead of TMA stores (diagnostics).
bool tma_store_disabled() {
    const char* e = getenv("VRWKV_NO_TMA_STORE");
    return e && e[0] && e[0] != '0';
}

// VRWKV_BWD_TMA_STORE=1 makes the backward kernel store gk, gv by TMA from
// shared memory; off by default: at two CTAs per SM, waiting for the bulk
// store to drain delays the next CTA more than the per-thread stores cost.
bool bwd_tma_store_enabled() {
    const char* e = getenv("VRWKV_BWD_TMA_STORE");
    return e && e[0] == '1' && e[1] == 0;
}

// VRWKV_TMA_CHUNK=8 keeps the forward TMA path on 8-token thread chunks even
// where the 16-token kernel qualifies (diagnostics and tests).
bool tma_chunk8_forced() {
    const char* e = getenv("VRWKV_TMA_CHUNK");
    return e && e[0] == '8' && e[1] == 0;
}

struct FastPlan {
    fast::Params p;
    bool tm;     // 32-token chunks with tensor-memory partial sums (biwkv_tm_kernel)
    bool rot;    // tm: rotated sub-chunk order (conflict-free shared-memory rows)
    int layout;
    int ntiles;  // tiles per CTA (sources, doubled with Q-Shift)
    bool qs;
    bool gx;  // exchange through the caller's workspace instead of a cluster
    int nt;   // threads per CTA
    int kl;   // tokens per thread chunk (8 or 16)
    dim3 grid;
    int smem;
};

// Workspace of the global-exchange path: 16 bytes of counters, then a flag
// per (column, rank), then a record per (column, rank); a column is one
// (batch row, 8-channel slab).
struct WsLayout {
    size_t flags_off, recs_off, bytes;
};
WsLayout ws_layout(int B, int C) {
    const size_t cols = (size_t)B * (size_t)((C + fast::kCS - 1) / fast::kCS);
    WsLayout L;
    L.flags_off = 16;
    L.recs_off = (L.flags_off + cols * fast::kClusterMax * sizeof(unsigned int) + 255) / 256 * 256;
    L.bytes = L.recs_off + cols * fast::kClusterMax * fast::kRecF4 * sizeof(float4);
    return L;
}

template <typename IO, int LAYOUT, bool QS, int NT, int KL, bool GX>
vrwkv_status launch_fast(const FastPlan& pl, cudaStream_t stream, bool* fell_back) {
    auto kern = fast::biwkv_tma_kernel<IO, LAYOUT, QS, NT, KL, GX>;
    static std::atomic<int> granted{0};
    static std::atomic<int> nonportable{0};
    cudaError_t e = ensure_smem(kern, granted, pl.smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    if (GX) {  // a plain 1-D grid: the CTAs of a column meet through the workspace
        cudaLaunchConfig_t gcfg = {};
        gcfg.gridDim = pl.grid;
        gcfg.blockDim = dim3(NT, 1, 1);
        gcfg.dynamicSmemBytes = pl.smem;
        gcfg.stream = stream;
        e = cudaLaunchKernelEx(&gcfg, kern, pl.p);
        if (e != cudaSuccess) return cuda_status(e, "biwkv_tma_kernel launch");
        g_last_kernel = "biwkv_tma_kernel";
        return ok();
    }
    if (pl.p.ncl > 8 && !nonportable.load()) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) {
            cudaGetLastError();
            *fell_back = true;
            return VRWKV_OK;
        }
        nonportable.store(1);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = pl.grid;
    cfg.blockDim = dim3(NT, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // let the hardware balance a cluster's CTAs over the SMs (measured with
    // 16-CTA clusters on the B200: 33 instead of 31 co-resident, 3 % faster)
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cluster_policy("VRWKV_CLUSTER_POLICY_NARROW");
    cfg.attrs = attr;
    cfg.numAttrs = pl.p.ncl > 1 ? 2 : 0;
    if (pl.p.ncl > 1) {
        // a cluster shape the GPU cannot co-schedule falls back to the generic kernel
        static std::atomic<int> checked[fast::kClusterMax + 1];
        int v = checked[pl.p.ncl].load();
        if (v == 0) {
            int n = 0;
            cudaError_t oe = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
            v = (oe == cudaSuccess && n > 0) ? 1 : -1;
            if (oe != cudaSuccess) cudaGetLastError();
            checked[pl.p.ncl].store(v);
        }
        if (v < 0) {
            *fell_back = true;
            return VRWKV_OK;
        }
    }
    e = cudaLaunchKernelEx(&cfg, kern, pl.p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_tma_kernel launch");
    g_last_kernel = "biwkv_tma_kernel";
    return ok();
}

template <typename IO, int NT, int KL, bool GX>
vrwkv_status dispatch_fast_nt(const FastPlan& pl, cudaStream_t s, bool* fb) {
    switch (pl.layout * 2 + (pl.qs ? 1 : 0)) {
    case fast::kKV * 2 + 0: return launch_fast<IO, fast::kKV, false, NT, KL, GX>(pl, s, fb);
    case fast::kKV * 2 + 1: return launch_fast<IO, fast::kKV, true, NT, KL, GX>(pl, s, fb);
    case fast::kRKV * 2 + 0: return launch_fast<IO, fast::kRKV, false, NT, KL, GX>(pl, s, fb);
    case fast::kRKV * 2 + 1: return launch_fast<IO, fast::kRKV, true, NT, KL, GX>(pl, s, fb);
    case fast::kX * 2 + 0: return launch_fast<IO, fast::kX, false, NT, KL, GX>(pl, s, fb);
    default: return launch_fast<IO, fast::kX, true, NT, KL, GX>(pl, s, fb);
    }
}

// CTA shapes of the fast path, two of 512 tokens x 8 channels at four CTAs
// per SM: 128 threads with 16-token chunks (the default: half the per-thread
// scan and exchange work per token), or 256 threads with 8-token chunks where
// a cluster's CTAs cannot hold whole 128-token warps; and one of 256 tokens
// (64 threads, 16-token chunks) for columns of at most 256 tokens, so a
// 14 x 14 grid keeps 13 of 16 chunks busy instead of 13 of 32 and its smaller
// tiles let twice the CTAs share an SM.
constexpr int kFastThreads16 = 128;
constexpr int kFastThreads8 = 256;
constexpr int kFastThreadsShort = 64;
constexpr int kFastTcMax = fast::Cfg<kFastThreads16, 16>::kTcMax;
constexpr int kFastTcShort = fast::Cfg<kFastThreadsShort, 16>::kTcMax;
static_assert(kFastTcMax == fast::Cfg<kFastThreads8, 8>::kTcMax, "one tile geometry for both long shapes");

// The 32-token tensor-memory kernel: a cluster per column as in the 8-channel
// kernel.  Sets *fell_back when the shape cannot be co-scheduled or more
// than four CTAs would share an SM (their tensor memory would not fit).
template <typename IO, int LAYOUT, bool QS, bool ROT, bool GX>
vrwkv_status launch_tm(const FastPlan& pl, cudaStream_t stream, bool* fell_back) {
    auto kern = tm32::biwkv_tm_kernel<IO, LAYOUT, QS, ROT, GX>;
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem(kern, granted, pl.smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = pl.grid;
    cfg.blockDim = dim3(tm32::kThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cluster_policy("VRWKV_CLUSTER_POLICY_TM");
    cfg.attrs = attr;
    cfg.numAttrs = (!GX && pl.p.ncl > 1) ? 2 : 0;  // GX: a plain 1-D grid of tickets
    // checked once per (cluster size, shared memory)
    static std::mutex mu;
    static std::vector<std::array<int, 3>> seen;
    int okv = 0;
    {
        std::lock_guard<std::mutex> lk(mu);
        for (const auto& a : seen)
            if (a[0] == pl.p.ncl && a[1] == pl.smem) okv = a[2];
    }
    if (okv == 0) {
        int per_sm = 0, nclu = 1;
        cudaError_t oe = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, tm32::kThreads, pl.smem);
        if (oe == cudaSuccess && !GX && pl.p.ncl > 1) oe = cudaOccupancyMaxActiveClusters(&nclu, kern, &cfg);
        if (oe != cudaSuccess) cudaGetLastError();
        okv = (oe == cudaSuccess && per_sm >= 1 && per_sm * tm32::kTmemCols <= 512 && nclu > 0) ? 1 : -1;
        std::lock_guard<std::mutex> lk(mu);
        seen.push_back({pl.p.ncl, pl.smem, okv});
    }
    if (okv < 0) {
        *fell_back = true;
        return VRWKV_OK;
    }
    e = cudaLaunchKernelEx(&cfg, kern, pl.p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_tm_kernel launch");
    g_last_kernel = "biwkv_tm_kernel";
    return ok();
}

template <typename IO, bool ROT, bool GX>
vrwkv_status dispatch_tm_layout(const FastPlan& pl, cudaStream_t s, bool* fb) {
    switch (pl.layout * 2 + (pl.qs ? 1 : 0)) {
    case fast::kKV * 2 + 0: return launch_tm<IO, fast::kKV, false, ROT, GX>(pl, s, fb);
    case fast::kKV * 2 + 1: return launch_tm<IO, fast::kKV, true, ROT, GX>(pl, s, fb);
    case fast::kRKV * 2 + 0: return launch_tm<IO, fast::kRKV, false, ROT, GX>(pl, s, fb);
    case fast::kRKV * 2 + 1: return launch_tm<IO, fast::kRKV, true, ROT, GX>(pl, s, fb);
    case fast::kX * 2 + 0: return launch_tm<IO, fast::kX, false, ROT, GX>(pl, s, fb);
    default: return launch_tm<IO, fast::kX, true, ROT, GX>(pl, s, fb);
    }
}

template <typename IO, bool ROT>
vrwkv_status dispatch_tm_rot(const FastPlan& pl, cudaStream_t s, bool* fb) {
    return pl.gx ? dispatch_tm_layout<IO, ROT, true>(pl, s, fb) : dispatch_tm_layout<IO, ROT, false>(pl, s, fb);
}

template <typename IO>
vrwkv_status dispatch_tm(const FastPlan& pl, cudaStream_t s, bool* fb) {
    // the rotated order is only ever planned for 16-byte rows (bfloat16)
    if constexpr (std::is_same<IO, __nv_bfloat16>::value) {
        if (pl.rot) return dispatch_tm_rot<IO, true>(pl, s, fb);
    }
    return dispatch_tm_rot<IO, false>(pl, s, fb);
}

template <typename IO>
vrwkv_status dispatch_fast(const FastPlan& pl, cudaStream_t s, bool* fb) {
    if (pl.nt == kFastThreadsShort) return dispatch_fast_nt<IO, kFastThreadsShort, 16, false>(pl, s, fb);
    if (pl.kl == 16)
        return pl.gx ? dispatch_fast_nt<IO, kFastThreads16, 16, true>(pl, s, fb)
                     : dispatch_fast_nt<IO, kFastThreads16, 16, false>(pl, s, fb);
    return pl.gx ? dispatch_fast_nt<IO, kFastThreads8, 8, true>(pl, s, fb)
                 : dispatch_fast_nt<IO, kFastThreads8, 8, false>(pl, s, fb);
}

// Shared memory of a fast-path CTA: the tiles (one extra for the gate
// factor when one x feeds r, k and v without Q-Shift) plus the scratch block.
int fast_smem(bool gate, bool qs, int ntiles, int tile_bytes, int nt) {
    const int nta = gate && !qs && ntiles == 1 ? ntiles + 1 : ntiles;
    const int scratch = nt == kFastThreadsShort ? (int)sizeof(fast::Scratch<kFastThreadsShort, 16>)
                        : nt == kFastThreads16  ? (int)sizeof(fast::Scratch<kFastThreads16, 16>)
                                                : (int)sizeof(fast::Scratch<kFastThreads8, 8>);
    return nta * tile_bytes + scratch + 128;  // + alignment slack
}

// VRWKV_QS_VIEW=flat takes Q-Shift through the flat token view wherever the
// TMA kernels run it (also where the image view qualifies), =image never
// (grids whose W is not a multiple of 8 then go to the generic kernel);
// diagnostics and tests.
int qs_view_forced() {
    const char* e = getenv("VRWKV_QS_VIEW");
    if (!e || !e[0]) return 0;
    return e[0] == 'f' ? 1 : (e[0] == 'i' ? -1 : 0);
}

// VRWKV_TM_IMAJ=0 keeps the tensor-memory kernel's tile loads on
// lane-strided boxes (eight or more per tile) instead of one residue-major
// box (diagnostics and tests).
bool tm_imaj_disabled() {
    const char* e = getenv("VRWKV_TM_IMAJ");
    return e && e[0] == '0' && e[1] == 0;
}

// VRWKV_TM_OSTORE=0 keeps the tensor-memory kernel's result stores at one
// lane-strided 256-token box each (diagnostics and tests).
bool tm_ofold_disabled() {
    const char* e = getenv("VRWKV_TM_OSTORE");
    return e && e[0] == '0' && e[1] == 0;
}

// VRWKV_SHORT_CTA=0 keeps columns of at most 256 tokens on the 512-token CTA
// shape (diagnostics and tests).
bool short_cta_disabled() {
    const char* e = getenv("VRWKV_SHORT_CTA");
    return e && e[0] == '0' && e[1] == 0;
}

// Shared memory of a tensor-memory kernel CTA: its tiles (one extra for the
// gate factor without Q-Shift), the scratch block, and at least the floor
// that keeps a fifth CTA off an SM.
int tm_smem(bool gate, bool qs, int ntiles, int tile_bytes, bool rot) {
    // one extra tile for the gate factor's second half when one x feeds r, k
    // and v without Q-Shift (one tile); separate r, k, v park it in k's slot
    const int nta = gate && !qs && ntiles == 1 ? ntiles + 1 : ntiles;
    const int stash = rot ? (int)sizeof(tm32::Stash) : 0;
    return std::max(nta * tile_bytes + (int)sizeof(tm32::Scratch) + stash + 128, tm32::kSmemFloor);
}

// VRWKV_TM_ROT=0 keeps the tensor-memory kernel's sub-chunks in natural order
// (diagnostics and tests).
bool tm_rot_disabled() {
    const char* e = getenv("VRWKV_TM_ROT");
    return e && e[0] == '0' && e[1] == 0;
}

// Rotated sub-chunk order where it pays: 16-byte token rows (bfloat16) and
// a stash that still leaves room for four CTAs per SM.
bool tm_rot_wanted(bool gate, bool qs, int ntiles, int tile_bytes, int es) {
    if (tm_rot_disabled() || es != 2) return false;
    return 4 * (tm_smem(gate, qs, ntiles, tile_bytes, true) + 1024) <= 228 * 1024;
}

// Plan the TMA path; returns false when the problem is outside its limits
// (the generic kernel then runs).  tmem_chunks plans the 32-token kernel
// (1024-token CTAs, clusters of up to 8).
bool plan_fast(FastPlan& pl, bool gate, const void* r, const void* k, const void* v, const float* w,
               const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
               const vrwkv_qshift_params* qs, void* ws, bool tmem_chunks = false) {
    if (tma_disabled()) return false;
    pl.tm = tmem_chunks;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const int es = elem_bytes(dtype);
    if (C % fast::kCS != 0 || !aligned(out, 16)) return false;
    const void* srcs[3];
    int nsrc;
    if (!gate) {
        pl.layout = fast::kKV;
        srcs[0] = k;
        srcs[1] = v;
        nsrc = 2;
    } else if (r == k && k == v) {
        pl.layout = fast::kX;
        srcs[0] = r;
        nsrc = 1;
    } else {
        pl.layout = fast::kRKV;
        srcs[0] = r;
        srcs[1] = k;
        srcs[2] = v;
        nsrc = 3;
    }
    for (int i = 0; i < nsrc; ++i)
        if (!aligned(srcs[i], 16)) return false;
    fast::Params& p = pl.p;
    pl.qs = qs != nullptr;
    p.B = B;
    p.T = T;
    p.C = C;
    const int RB = fast::kCS * es;
    const int ntiles = nsrc * (pl.qs ? 2 : 1);
    pl.ntiles = ntiles;
    const bool short_cta = !pl.tm && T <= kFastTcShort && !tma_chunk8_forced() && !short_cta_disabled();
    const int TcMax = pl.tm ? tm32::kTc : (short_cta ? kFastTcShort : kFastTcMax);
    pl.kl = pl.tm ? tm32::kKL : (tma_chunk8_forced() ? 8 : 16);
    p.flat = 0;
    if (pl.qs) {
        p.H = qs->H;
        p.W = qs->W;
        p.s = qs->shift_pixel;
        p.g = qs_bounds(C, qs->gamma);
        p.ng = shifted_groups(qs);
        if (!bounds_multiple_of(p.g, fast::kCS)) return false;
        // the image view (C, W, H, B) needs W a multiple of 8 and at most 256
        // (one box row); any other W takes the flat token view
        const int view = qs_view_forced();
        p.flat = (view > 0 || p.W > 256 || p.W % fast::kL != 0) ? 1 : 0;
        if (p.flat && view < 0) return false;
    }
    if (pl.qs && !p.flat) {
        if (T <= TcMax) {
            p.rows = p.H;
            p.Tc = T;
            p.ncl = 1;
        } else {
            // whole image rows per CTA, a whole number of warps' tokens:
            // 16-token chunks where possible, else 8-token chunks
            int rows = 0;
            for (int kl = pl.kl; kl >= 8 && rows == 0; kl /= 2) {
                if (pl.tm && kl != tm32::kKL) break;
                const int warp_tok = kl == 32   ? tm32::kWarpTok
                                     : kl == 16 ? fast::Cfg<kFastThreads16, 16>::kWarpTok
                                                : fast::Cfg<kFastThreads8, 8>::kWarpTok;
                for (int rr = TcMax / p.W; rr >= 1; --rr)
                    if ((rr * p.W) % warp_tok == 0) {
                        rows = rr;
                        pl.kl = kl;
                        break;
                    }
            }
            if (rows == 0 || rows > 256) {
                // whole image rows cannot make whole warps: the flat view
                if (qs_view_forced() < 0) return false;
                p.flat = 1;
            } else {
                p.rows = rows;
                p.Tc = rows * p.W;
                p.ncl = (p.H + rows - 1) / rows;
            }
        }
    }
    if (!pl.qs || p.flat) {
        if (!pl.qs) {
            p.H = 1;
            p.W = T;
            p.s = 0;
            p.g = no_shift_bounds();
            p.ng = 4;
        }
        p.rows = 1;
        p.Tc = std::min(T, TcMax);
        p.ncl = (T + p.Tc - 1) / p.Tc;
    }
    if (p.ncl > (pl.tm ? tm32::kClusterMax : fast::kClusterMax)) return false;
    // 8 sub-tiles of TcMax / 8 token rows; every thread reads its row of
    // each, so a tile always spans TcMax tokens even when the boxes deliver
    // fewer
    p.tile_bytes = TcMax * RB;
    // a sub-tile receives (W / 8) x rows token rows with Q-Shift in the image
    // view (one box), and its full TcMax / 8 rows in the flat view (boxes of
    // 32 rows; tokens past T arrive as zeros)
    p.box_bytes = (pl.qs && !p.flat ? (p.W / fast::kL) * p.rows : TcMax / fast::kL) * RB;
    pl.nt = pl.tm ? tm32::kThreads : (short_cta ? kFastThreadsShort : (pl.kl == 16 ? kFastThreads16 : kFastThreads8));
    pl.rot = pl.tm && tm_rot_wanted(gate, pl.qs, ntiles, p.tile_bytes, es);
    pl.smem = pl.tm ? tm_smem(gate, pl.qs, ntiles, p.tile_bytes, pl.rot) : fast_smem(gate, pl.qs, ntiles, p.tile_bytes, pl.nt);
    if (pl.smem > 227 * 1024) return false;
    const CUtensorMapDataType dt =
        dtype == VRWKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t ces = (cuuint64_t)C * es;  // bytes per token
    auto encode = [&](CUtensorMap* m, const void* src, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
                      const cuuint32_t* box, const cuuint32_t* estr, CUtensorMapL2promotion l2) {
        return enc(m, dt, rank, const_cast<void*>(src), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_NONE, l2, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    };
    const auto l2_in = CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
    const auto l2_out = CU_TENSOR_MAP_L2_PROMOTION_NONE;
    // Lane-strided views (element stride 8 along the tokens: lane i's box
    // holds tokens 8 m + i): the image (C, W, H, B) with boxes of `rows` image
    // rows, and the flat tokens (C, T, B) with boxes of 256 tokens.
    auto image_strided = [&](CUtensorMap* m, const void* src, int rows) {
        const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)p.W, (cuuint64_t)p.H, (cuuint64_t)B};
        const cuuint64_t strides[3] = {ces, (cuuint64_t)p.W * ces, (cuuint64_t)p.H * p.W * ces};
        const cuuint32_t box[4] = {(cuuint32_t)fast::kCS, (cuuint32_t)p.W, (cuuint32_t)rows, 1};
        const cuuint32_t estr[4] = {1, (cuuint32_t)fast::kL, 1, 1};
        return encode(m, src, 4, dims, strides, box, estr, l2_in);
    };
    auto flat_strided = [&](CUtensorMap* m, const void* src, CUtensorMapL2promotion l2) {
        const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
        const cuuint64_t strides[2] = {ces, (cuuint64_t)T * ces};
        const cuuint32_t box[3] = {(cuuint32_t)fast::kCS, 256u, 1};
        const cuuint32_t estr[3] = {1, (cuuint32_t)fast::kL, 1};
        return encode(m, src, 3, dims, strides, box, estr, l2);
    };
    // Residue-major views for the tensor-memory kernel (T a multiple of 8):
    // the tokens as (C, T / 8, 8, B), token 8 m + i at (m, i), and the image
    // as (C, W / 8, H, 8, B); the residue axis is outermost in the box, so one
    // box fills all eight sub-tiles of a tile (128 rows each).
    auto flat_residue = [&](CUtensorMap* m, const void* src, CUtensorMapL2promotion l2) {
        const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)T / 8, 8, (cuuint64_t)B};
        const cuuint64_t strides[3] = {8 * ces, ces, (cuuint64_t)T * ces};
        const cuuint32_t box[4] = {(cuuint32_t)fast::kCS, (cuuint32_t)(tm32::kTc / 8), 8, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        return encode(m, src, 4, dims, strides, box, estr, l2);
    };
    auto image_residue = [&](CUtensorMap* m, const void* src) {
        const cuuint64_t dims[5] = {(cuuint64_t)C, (cuuint64_t)p.W / 8, (cuuint64_t)p.H, 8, (cuuint64_t)B};
        const cuuint64_t strides[4] = {8 * ces, (cuuint64_t)p.W * ces, ces, (cuuint64_t)p.H * p.W * ces};
        const cuuint32_t box[5] = {(cuuint32_t)fast::kCS, (cuuint32_t)(p.W / 8), (cuuint32_t)p.rows, 8, 1};
        const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
        return encode(m, src, 5, dims, strides, box, estr, l2_in);
    };
    const bool img = pl.qs && !p.flat;
    p.imaj = 0;
    p.nbox = pl.tm && !img ? tm32::kNW : 1;
    if (pl.tm && !tm_imaj_disabled() && T % 8 == 0 && (!img || p.rows * p.W == tm32::kTc)) {
        bool okm = true;
        for (int i = 0; i < nsrc && okm; ++i) {
            okm = img ? image_residue(&p.map[i], srcs[i]) : flat_residue(&p.map[i], srcs[i], l2_in);
            if (okm && pl.qs) okm = img ? image_strided(&p.xmap[i], srcs[i], p.rows) : flat_strided(&p.xmap[i], srcs[i], l2_in);
        }
        if (okm) {
            p.imaj = 1;
            p.nbox = 1;
        }
    }
    if (!p.imaj) {
        for (int i = 0; i < nsrc; ++i) {
            const bool okm = img ? image_strided(&p.map[i], srcs[i], p.rows) : flat_strided(&p.map[i], srcs[i], l2_in);
            if (!okm) return false;
        }
    }
    // The output in the tiles' layout: lane-strided boxes of 256 tokens; a
    // CTA stores by TMA when its span is whole boxes or ends the column, so no
    // box reaches another CTA's tokens (the tensor bound clips at T).  The
    // tensor-memory kernel stores through the residue-major view instead, one
    // box for its 1024 tokens, where T is a multiple of 8 and a CTA spans 1024
    // tokens or the whole column.
    p.ofold = pl.tm && T % 8 == 0 && (p.Tc == tm32::kTc || p.ncl == 1) && !tm_ofold_disabled() ? 1 : 0;
    bool okout = p.ofold ? flat_residue(&p.omap, out, l2_out) : flat_strided(&p.omap, out, l2_out);
    if (!okout && p.ofold) {
        p.ofold = 0;
        okout = flat_strided(&p.omap, out, l2_out);
    }
    p.tma_store = (okout && (p.Tc % 256 == 0 || p.ncl == 1) && !tma_store_disabled()) ? 1 : 0;
    p.invT = (float)(1.0 / (double)T);
    p.err = device_error_word();
    if (!p.err) return false;
    p.w = w;
    p.u = u;
    p.mu[0] = qs ? qs->mu_r : nullptr;
    p.mu[1] = qs ? qs->mu_k : nullptr;
    p.mu[2] = qs ? qs->mu_v : nullptr;
    p.out = static_cast<char*>(out);
    pl.grid = dim3(p.ncl, C / fast::kCS, B);
    p.nslab = C / fast::kCS;
    p.total = p.ncl * p.nslab * B;
    pl.gx = ws != nullptr && p.ncl > 1;
    if (pl.tm && !p.tma_store) return false;
    if (pl.gx) {
        const WsLayout L = ws_layout(B, C);
        char* base = static_cast<char*>(ws);
        p.ws_ctl = reinterpret_cast<unsigned int*>(base);
        p.ws_flag = reinterpret_cast<unsigned int*>(base + L.flags_off);
        p.ws_rec = reinterpret_cast<float4*>(base + L.recs_off);
        pl.grid = dim3((unsigned)p.total, 1, 1);
    } else {
        p.ws_ctl = p.ws_flag = nullptr;
        p.ws_rec = nullptr;
    }
    return true;
}

// ---------------------------------------------------------------------------
// 16-channel slab path (biwkv_wide_kernel): long sequences through a workspace,
// and VRWKV_FORWARD=wide
// ---------------------------------------------------------------------------
bool wide_disabled() {
    const char* e = getenv("VRWKV_DISABLE_WIDE");
    return e && e[0] == '1';
}

// Which kernel serves sequences of up to 4096 tokens when both qualify:
// the 8-channel kernel unless VRWKV_FORWARD=wide.
bool wide_preferred() {
    const char* e = getenv("VRWKV_FORWARD");
    return e && e[0] == 'w';
}

// The 32-token tensor-memory kernel takes columns of more than 512 tokens,
// which the 8-channel kernel would split over a cluster (measured on the
// B200 at C = 1024: 91.0 against 112.2 us at T = 768, 76.2 against 94.4 us
// at T = 1024, but 105.3 against 64.0 us at T = 512, where the 8-channel
// kernel needs one CTA and most tensor-memory threads have no token);
// VRWKV_FORWARD=tm takes it wherever it qualifies, VRWKV_FORWARD=narrow
// never.
bool tm_wanted(int T) {
    const char* e = getenv("VRWKV_FORWARD");
    if (e && e[0] == 't') return true;
    if (e && e[0]) return false;
    return T > 512;
}

struct WidePlan {
    wide::Params p;
    int layout;
    bool qs;
    bool seg;  // segmented columns: clusters meet through the workspace
    dim3 grid;
    int smem;
};

// Workspace of the segmented 16-channel path: 16 bytes of counters, a flag
// per (column, segment), then a record (three float4) per (column, segment,
// channel pair); a column is one (batch row, 16-channel slab).
constexpr int kWideSegTokens = wide::kTc * wide::kClusterMax;  // tokens per segment (one cluster)
constexpr int kWideSegMax = 8;                                  // segments per column (T <= 32768)
WsLayout wide_ws_layout(int B, int T, int C) {
    const size_t cols = (size_t)B * (size_t)(C / wide::kCW);
    const size_t nseg = (size_t)((T + kWideSegTokens - 1) / kWideSegTokens);
    WsLayout L;
    L.flags_off = 16;
    L.recs_off = (L.flags_off + cols * nseg * sizeof(unsigned int) + 255) / 256 * 256;
    L.bytes = L.recs_off + cols * nseg * wide::kNP * 3 * sizeof(float4);
    return L;
}

// Plan the 16-channel slab kernel; false when the shape does not qualify
// (the caller then takes another path).
bool plan_wide(WidePlan& pl, bool gate, const void* r, const void* k, const void* v, const float* w,
               const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
               void* ws = nullptr, size_t ws_bytes = 0) {
    if (tma_disabled() || wide_disabled() || tma_chunk8_forced()) return false;
    const int es = elem_bytes(dtype);
    if (C % wide::kCW != 0 || T % wide::kL != 0 || B > 65535 || C / wide::kCW > 65535) return false;
    // one cluster per column up to 4096 tokens; longer columns split into
    // segments of one cluster each, which meet through the workspace
    pl.seg = T > kWideSegTokens;
    const int ncl = pl.seg ? wide::kClusterMax : (T + wide::kTc - 1) / wide::kTc;
    const int nseg = pl.seg ? (T + kWideSegTokens - 1) / kWideSegTokens : 1;
    if (nseg > kWideSegMax) return false;
    if (pl.seg && (!ws || ws_bytes < wide_ws_layout(B, T, C).bytes)) return false;
    if ((long long)B * (C / wide::kCW) * nseg > 65535) return false;
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    wide::Params& p = pl.p;
    p = wide::Params{};
    pl.qs = qs != nullptr;
    p.qs = pl.qs ? 1 : 0;
    p.W = pl.qs ? qs->W : T;
    p.s = pl.qs ? qs->shift_pixel : 0;
    p.g = pl.qs ? qs_bounds(C, qs->gamma) : no_shift_bounds();
    p.ng = shifted_groups(qs);
    p.hv = 0;
    if (pl.qs && p.s > 0) {
        if (!bounds_multiple_of(p.g, wide::kCW) || p.W % wide::kL != 0) return false;
        // horizontal groups need shift 1 (the neighbour is the adjacent
        // token); vertical groups read a halo of s*W tokens
        const bool horiz = p.g.b[0] > 0 || p.g.b[1] > p.g.b[0];
        const bool vert = p.ng > 2 && (p.g.b[2] > p.g.b[1] || p.g.b[3] > p.g.b[2]);
        if (horiz && p.s != 1) return false;
        if (vert) {
            const long long hv = (long long)p.s * p.W / wide::kL;
            if (hv > wide::kHaloMax) return false;
            p.hv = (int)hv;
        }
    }
    const void* srcs[3];
    int nsrc;
    if (!gate) {
        pl.layout = wide::kKV;
        srcs[0] = k;
        srcs[1] = v;
        nsrc = 2;
    } else if (r == k && k == v) {
        pl.layout = wide::kX;
        srcs[0] = r;
        nsrc = 1;
    } else {
        pl.layout = wide::kRKV;
        srcs[0] = r;
        srcs[1] = k;
        srcs[2] = v;
        nsrc = 3;
    }
    for (int i = 0; i < nsrc; ++i)
        if (!aligned(srcs[i], 16)) return false;
    if (!aligned(out, 16) || ((size_t)C * es) % 16 != 0) return false;
    const CUtensorMapDataType dt = dtype == VRWKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    for (int i = 0; i < nsrc; ++i) {
        // (C, 16, T/16, B): channel, token within a 16-token chunk, chunk,
        // batch row; a box of 17 rows per chunk (the 17th outside the view,
        // zero-filled) spaces the chunks in shared memory
        const cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)wide::kL, (cuuint64_t)(T / wide::kL), (cuuint64_t)B};
        const cuuint64_t strides[3] = {(cuuint64_t)C * es, (cuuint64_t)C * es * wide::kL, (cuuint64_t)T * C * es};
        const cuuint32_t box[4] = {(cuuint32_t)wide::kCW, (cuuint32_t)wide::kRows, (cuuint32_t)wide::kBoxChunks, 1};
        const cuuint32_t estr[4] = {1, 1, 1, 1};
        const CUresult cr = enc(&p.map[i], dt, 4, const_cast<void*>(srcs[i]), dims, strides, box, estr,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (cr != CUDA_SUCCESS) return false;
    }
    p.err = device_error_word();
    if (!p.err) return false;
    p.w = w;
    p.u = u;
    p.mu[0] = qs ? qs->mu_r : nullptr;
    p.mu[1] = qs ? qs->mu_k : nullptr;
    p.mu[2] = qs ? qs->mu_v : nullptr;
    p.out = static_cast<char*>(out);
    p.B = B;
    p.T = T;
    p.C = C;
    p.invT = (float)(1.0 / (double)T);
    p.nchunkT = T / wide::kL;
    p.ncl = ncl;
    p.nseg = nseg;
    p.nslab = C / wide::kCW;
    p.total = ncl * nseg * B * p.nslab;
    if (pl.seg) {
        const WsLayout L = wide_ws_layout(B, T, C);
        char* base = static_cast<char*>(ws);
        p.ws_ctl = reinterpret_cast<unsigned int*>(base);
        p.ws_flag = reinterpret_cast<unsigned int*>(base + L.flags_off);
        p.ws_rec = reinterpret_cast<float4*>(base + L.recs_off);
    }
    // shared memory: scratch, the widest tile (main chunks + halo boxes) per
    // source, the parked gate factors
    const int halo4 = pl.qs ? (std::max(p.hv, 1) + wide::kBoxChunks - 1) / wide::kBoxChunks * wide::kBoxChunks : 0;
    const int tile = (wide::kChunks + halo4) * wide::kRows * wide::kCW * es;
    const int park = gate ? wide::kTc * wide::kNP * (int)sizeof(float2) : 0;
    pl.smem = (int)((sizeof(wide::Scratch) + 127) / 128 * 128) + nsrc * tile + park + 128;
    if (pl.smem > 227 * 1024) return false;
    pl.grid = pl.seg ? dim3(ncl, (unsigned)(nseg * B * p.nslab), 1) : dim3(ncl, C / wide::kCW, B);
    return true;
}

template <typename IO, int LAYOUT, bool QS, bool SEG>
vrwkv_status launch_wide(const WidePlan& pl, cudaStream_t stream, bool* fell_back) {
    auto kern = wide::biwkv_wide_kernel<IO, LAYOUT, QS, SEG>;
    static std::atomic<int> granted{0};
    cudaError_t e = ensure_smem(kern, granted, pl.smem);
    if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = pl.grid;
    cfg.blockDim = dim3(wide::kThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    cfg.attrs = attr;
    cfg.numAttrs = pl.p.ncl > 1 ? 2 : 0;
    if (pl.p.ncl > 1) {
        static std::atomic<int> checked[wide::kClusterMax + 1];
        int v = checked[pl.p.ncl].load();
        if (v == 0) {
            int n = 0;
            cudaError_t oe = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
            v = (oe == cudaSuccess && n > 0) ? 1 : -1;
            if (oe != cudaSuccess) cudaGetLastError();
            checked[pl.p.ncl].store(v);
        }
        if (v < 0) {
            *fell_back = true;
            return VRWKV_OK;
        }
    }
    e = cudaLaunchKernelEx(&cfg, kern, pl.p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_wide_kernel launch");
    g_last_kernel = "biwkv_wide_kernel";
    return ok();
}

template <typename IO, bool SEG>
vrwkv_status dispatch_wide_seg(const WidePlan& pl, cudaStream_t s, bool* fb) {
    switch (pl.layout * 2 + (pl.qs ? 1 : 0)) {
    case wide::kKV * 2 + 0: return launch_wide<IO, wide::kKV, false, SEG>(pl, s, fb);
    case wide::kKV * 2 + 1: return launch_wide<IO, wide::kKV, true, SEG>(pl, s, fb);
    case wide::kRKV * 2 + 0: return launch_wide<IO, wide::kRKV, false, SEG>(pl, s, fb);
    case wide::kRKV * 2 + 1: return launch_wide<IO, wide::kRKV, true, SEG>(pl, s, fb);
    case wide::kX * 2 + 0: return launch_wide<IO, wide::kX, false, SEG>(pl, s, fb);
    default: return launch_wide<IO, wide::kX, true, SEG>(pl, s, fb);
    }
}

template <typename IO>
vrwkv_status dispatch_wide(const WidePlan& pl, cudaStream_t s, bool* fb) {
    return pl.seg ? dispatch_wide_seg<IO, true>(pl, s, fb) : dispatch_wide_seg<IO, false>(pl, s, fb);
}

vrwkv_status check_qs(const vrwkv_qshift_params* qs, int T, int C) {
    if (qs->mode != VRWKV_QSHIFT_QUAD && qs->mode != VRWKV_QSHIFT_BIDIR)
        return fail(VRWKV_ERR_INVALID_ARG, "qs: unknown mode %d", qs->mode);
    if (qs->H <= 0 || qs->W <= 0) return fail(VRWKV_ERR_INVALID_ARG, "qs: H and W must be positive");
    if ((long long)qs->H * qs->W != T)
        return fail(VRWKV_ERR_INVALID_ARG, "qs: H*W (%lld) must equal T (%d)",
                    (long long)qs->H * qs->W, T);
    if (qs->shift_pixel < 0) return fail(VRWKV_ERR_INVALID_ARG, "qs: shift_pixel must be >= 0");
    if (!(qs->gamma >= 0.0 && qs->gamma <= 0.25))
        return fail(VRWKV_ERR_INVALID_ARG, "qs: gamma must lie in [0, 1/4]");
    const float* mus[3] = {qs->mu_r, qs->mu_k, qs->mu_v};
    for (const float* m : mus)
        if (m && !aligned(m, 4)) return fail(VRWKV_ERR_INVALID_ARG, "qs: mu must be 4-byte aligned");
    (void)C;
    return VRWKV_OK;
}

// Shared front end of vrwkv_biwkv_fwd (gate = false) and vrwkv_spatial_gate.
vrwkv_status fused_entry(bool gate, const void* r, const void* k, const void* v, const float* w,
                         const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
                         const vrwkv_qshift_params* qs, void* stream, bool with_ws = false,
                         void* ws = nullptr, size_t ws_bytes = 0) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!k || !v || !w || !u || !out || (gate && !r))
        return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    const int es = elem_bytes(dtype);
    const void* toks[3] = {gate ? r : nullptr, k, v};
    for (const void* t : toks)
        if (t && !aligned(t, es)) return fail(VRWKV_ERR_INVALID_ARG, "token tensor misaligned");
    if (!aligned(out, es)) return fail(VRWKV_ERR_INVALID_ARG, "output misaligned");
    if (!aligned(w, 4) || !aligned(u, 4)) return fail(VRWKV_ERR_INVALID_ARG, "w/u misaligned");
    if (qs) {
        vrwkv_status st = check_qs(qs, T, C);
        if (st != VRWKV_OK) return st;
    }
    const size_t nbytes = (size_t)B * T * C * es;
    for (const void* t : toks)
        if (overlaps(out, nbytes, t, nbytes)) return fail(VRWKV_ERR_INVALID_ARG, "output overlaps an input");
    if (overlaps(out, nbytes, w, (size_t)C * 4) || overlaps(out, nbytes, u, (size_t)C * 4))
        return fail(VRWKV_ERR_INVALID_ARG, "output overlaps w or u");
    if (qs) {
        const float* mus[3] = {qs->mu_r, qs->mu_k, qs->mu_v};
        for (const float* m : mus)
            if (overlaps(out, nbytes, m, (size_t)C * 4))
                return fail(VRWKV_ERR_INVALID_ARG, "output overlaps a mu vector");
    }

    if (with_ws) {
        if (!ws) return fail(VRWKV_ERR_INVALID_ARG, "workspace is NULL");
        if (!aligned(ws, 256)) return fail(VRWKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
        const size_t need = ws_layout(B, C).bytes;
        if (ws_bytes < need)
            return fail(VRWKV_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed", ws_bytes,
                        need);
        for (const void* t : toks)
            if (overlaps(ws, need, t, nbytes)) return fail(VRWKV_ERR_INVALID_ARG, "workspace overlaps an input");
        if (overlaps(ws, need, out, nbytes)) return fail(VRWKV_ERR_INVALID_ARG, "workspace overlaps the output");
    }
    // the 16-channel kernel: one cluster per column up to 4096 tokens; with
    // a workspace, longer columns in segments that meet through it (shorter
    // ones keep the 8-channel global-exchange path the workspace names)
    if (with_ws ? T > kWideSegTokens : (T <= kWideSegTokens && wide_preferred())) {
        WidePlan wp;
        if (plan_wide(wp, gate, r, k, v, w, u, out, B, T, C, dtype, qs, with_ws ? ws : nullptr, ws_bytes)) {
            bool fell_back = false;
            cudaStream_t ws_ = static_cast<cudaStream_t>(stream);
            vrwkv_status st = dtype == VRWKV_F32 ? dispatch_wide<float>(wp, ws_, &fell_back)
                                                 : dispatch_wide<__nv_bfloat16>(wp, ws_, &fell_back);
            if (!fell_back) return st;
        }
    }
    // the 32-token kernel: a cluster per column, or with a workspace (T <= 4096
    // here; longer ones took the 16-channel segments above) its global exchange
    if (B <= 65535 && C / vrwkv::fast::kCS <= 65535 && tm_wanted(T)) {
        FastPlan fp;
        if (plan_fast(fp, gate, r, k, v, w, u, out, B, T, C, dtype, qs, with_ws ? ws : nullptr, true)) {
            bool fell_back = false;
            cudaStream_t fs = static_cast<cudaStream_t>(stream);
            vrwkv_status st = dtype == VRWKV_F32 ? dispatch_tm<float>(fp, fs, &fell_back)
                                                 : dispatch_tm<__nv_bfloat16>(fp, fs, &fell_back);
            if (!fell_back) return st;
        }
    }
    if (B <= 65535 && C / vrwkv::fast::kCS <= 65535) {
        FastPlan fp;
        if (plan_fast(fp, gate, r, k, v, w, u, out, B, T, C, dtype, qs, with_ws ? ws : nullptr)) {
            bool fell_back = false;
            cudaStream_t fs = static_cast<cudaStream_t>(stream);
            vrwkv_status st = dtype == VRWKV_F32 ? dispatch_fast<float>(fp, fs, &fell_back)
                                                 : dispatch_fast<__nv_bfloat16>(fp, fs, &fell_back);
            if (!fell_back) return st;
        }
    }

    FusedPlan pl{};
    FusedParams& p = pl.p;
    const int slabs = (C + kCS - 1) / kCS;
    if (B > 65535 || slabs > 65535)
        return fail(VRWKV_ERR_UNSUPPORTED, "B (%d) or C/16 (%d) exceeds the grid limit 65535", B, slabs);
    if (T <= kTcMax) {
        p.ncl = 1;
        p.Tc = T;
    } else {
        p.ncl = (T + kTcMax - 1) / kTcMax;
        if (p.ncl > kClusterMax)
            return fail(VRWKV_ERR_UNSUPPORTED, "T = %d exceeds the supported maximum %d", T,
                        kTcMax * kClusterMax);
        p.Tc = ((T + p.ncl - 1) / p.ncl + 31) / 32 * 32;
    }
    pl.qs = qs != nullptr;
    if (pl.qs && p.ncl > 1) {
        long long halo = (long long)qs->shift_pixel * qs->W;
        p.halo = (int)std::min<long long>(halo, T);
    } else {
        p.halo = 0;
    }
    p.rows = p.Tc + 2 * p.halo;
    const int pitch = kCS * es;
    p.tile_bytes = ((padded_row(p.rows - 1) + 1) * pitch + 127) / 128 * 128;
    if (!gate) {
        pl.layout = kKV;
        p.src[0] = static_cast<const char*>(k);
        p.src[1] = static_cast<const char*>(v);
        pl.ntiles = 2;
    } else if (r == k && k == v) {
        pl.layout = kX;
        p.src[0] = static_cast<const char*>(r);
        pl.ntiles = 1;
    } else {
        pl.layout = kRKV;
        p.src[0] = static_cast<const char*>(r);
        p.src[1] = static_cast<const char*>(k);
        p.src[2] = static_cast<const char*>(v);
        pl.ntiles = 3;
    }
    pl.smem = pl.ntiles * p.tile_bytes + (int)sizeof(Scratch);
    if (pl.smem > 227 * 1024)
        return fail(VRWKV_ERR_UNSUPPORTED,
                    "Q-Shift halo of %d tokens needs %d bytes of shared memory (limit %d)", p.halo,
                    pl.smem, 227 * 1024);
    p.w = w;
    p.u = u;
    p.mu_r = qs ? qs->mu_r : nullptr;
    p.mu_k = qs ? qs->mu_k : nullptr;
    p.mu_v = qs ? qs->mu_v : nullptr;
    p.out = static_cast<char*>(out);
    p.B = B;
    p.T = T;
    p.C = C;
    p.H = qs ? qs->H : 1;
    p.W = qs ? qs->W : T;
    p.s = qs ? qs->shift_pixel : 0;
    p.g = qs ? qs_bounds(C, qs->gamma) : no_shift_bounds();
    p.ng = shifted_groups(qs);
    bool vin = ((size_t)C * es) % 16 == 0;
    for (int i = 0; i < pl.ntiles; ++i) vin = vin && aligned(p.src[i], 16);
    p.vec_in = vin ? 1 : 0;
    p.vec_out = (C % 2 == 0 && aligned(out, 2 * es)) ? 1 : 0;
    const int nch = (p.Tc + kL - 1) / kL;
    pl.threads = std::max(kMinThreads, (kNP * nch + 31) / 32 * 32);
    pl.grid = dim3(p.ncl, slabs, B);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return dtype == VRWKV_F32 ? dispatch_layout<float>(pl, s) : dispatch_layout<__nv_bfloat16>(pl, s);
}

// ---------------------------------------------------------------------------
// Host-buffer front end of vrwkv_spatial_gate: the batch is cut into slices
// of slice_b rows (every (b, c) column is independent and Q-Shift mixes
// tokens of one batch row only, so a slice is an exact sub-problem); slice i
// is copied host -> device into slot i % 2 of the caller's device buffer on a
// copy-in stream, computed on the caller's stream and copied back on a
// copy-out stream, so the two copy directions and the kernels overlap.
// ---------------------------------------------------------------------------
size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

// Device slots of the host pipeline (staging for one slice each).
constexpr int kHostSlots = 3;

size_t host_slot_bytes(int slice_b, int T, int C, int es, int inputs) {
    const size_t tensor = (size_t)slice_b * T * C * es;
    return (size_t)(inputs + 1) * round256(tensor);
}

// Streams and events of the pipeline, created once per device (never freed:
// they live as long as the process, like the library's other per-device
// state).  A mutex serialises the enqueueing of calls from different host
// threads onto them.
struct HostPipe {
    cudaStream_t in = nullptr, outs = nullptr;
    cudaEvent_t start = nullptr, loaded[kHostSlots] = {}, done[kHostSlots] = {}, freed[kHostSlots] = {};
    bool ok = false;
};

HostPipe* host_pipe(int dev) {
    static std::mutex mu;
    static HostPipe pipes[64];
    std::lock_guard<std::mutex> g(mu);
    if (dev < 0 || dev >= 64) return nullptr;
    HostPipe& p = pipes[dev];
    if (!p.ok) {
        bool good = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&p.outs, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&p.start, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; i < kHostSlots && good; ++i)
            good = cudaEventCreateWithFlags(&p.loaded[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&p.freed[i], cudaEventDisableTiming) == cudaSuccess;
        if (!good) return nullptr;
        p.ok = true;
    }
    return &p;
}

std::mutex& host_pipe_enqueue_mutex() {
    static std::mutex mu;
    return mu;
}

bool host_pinned(const void* p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

vrwkv_status host_pipeline(const void* r, const void* k, const void* v, const float* w, const float* u,
                           void* out, int B, int T, int C, vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
                           int slice_b, void* dev_buf, size_t dev_buf_bytes, cudaStream_t s) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!r || !k || !v || !w || !u || !out || !dev_buf)
        return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    if (slice_b <= 0 || slice_b > B)
        return fail(VRWKV_ERR_INVALID_ARG, "slice_b must lie in [1, B] (got %d)", slice_b);
    const int es = elem_bytes(dtype);
    // distinct host inputs: r, k, v may be one buffer (copied once)
    const void* srcs[3] = {k, v, r};
    int slot_of[3] = {0, 0, 0};
    int inputs = 0;
    for (int i = 0; i < 3; ++i) {
        int found = -1;
        for (int j = 0; j < i; ++j)
            if (srcs[j] == srcs[i]) found = slot_of[j];
        slot_of[i] = found >= 0 ? found : inputs++;
    }
    const size_t tensor_full = (size_t)B * T * C * es;
    for (int i = 0; i < 3; ++i)
        if (overlaps(out, tensor_full, srcs[i], tensor_full))
            return fail(VRWKV_ERR_INVALID_ARG, "out overlaps an input");
    const size_t slot = host_slot_bytes(slice_b, T, C, es, inputs);
    if (dev_buf_bytes < 2 * slot)
        return fail(VRWKV_ERR_INVALID_ARG, "device buffer holds %zu bytes; slices of %d rows need %zu",
                    dev_buf_bytes, slice_b, 2 * slot);
    // as many slots as the buffer holds, up to three: with three, a slice's
    // copy in never waits for the copy out of the slice two before it
    const int nslots = (int)std::min<size_t>(kHostSlots, dev_buf_bytes / slot);
    if (!aligned(dev_buf, 256)) return fail(VRWKV_ERR_INVALID_ARG, "device buffer must be 256-byte aligned");
    for (const void* p : {r, k, v, (const void*)out})
        if (!host_pinned(p))
            return fail(VRWKV_ERR_INVALID_ARG, "host buffers must be page-locked (cudaHostAlloc / cudaHostRegister)");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cuda_status(cudaGetLastError(), "cudaGetDevice");
    HostPipe* hp = host_pipe(dev);
    if (!hp) return fail(VRWKV_ERR_CUDA, "cannot create the copy streams");
    std::lock_guard<std::mutex> guard(host_pipe_enqueue_mutex());

    const size_t row = (size_t)T * C * es;  // bytes of one batch row
    const size_t part = round256((size_t)slice_b * row);
    char* base = static_cast<char*>(dev_buf);
    auto in_ptr = [&](int sl, int i) { return base + sl * slot + (size_t)slot_of[i] * part; };
    auto out_ptr = [&](int sl) { return base + sl * slot + (size_t)inputs * part; };
    auto check = [&](cudaError_t e, const char* what) -> bool {
        if (e == cudaSuccess) return true;
        cuda_status(e, what);
        return false;
    };
    // the pipeline starts after the work already queued on the caller's stream
    if (!check(cudaEventRecord(hp->start, s), "event record") ||
        !check(cudaStreamWaitEvent(hp->in, hp->start, 0), "stream wait") ||
        !check(cudaStreamWaitEvent(hp->outs, hp->start, 0), "stream wait"))
        return VRWKV_ERR_CUDA;
    const int nslices = (B + slice_b - 1) / slice_b;
    for (int i = 0; i < nslices; ++i) {
        const int sl = i % nslots;
        const int b0 = i * slice_b, nb = std::min(slice_b, B - b0);
        const size_t off = (size_t)b0 * row, n = (size_t)nb * row;
        if (i >= nslots && !check(cudaStreamWaitEvent(hp->in, hp->freed[sl], 0), "stream wait"))
            return VRWKV_ERR_CUDA;
        for (int j = 0; j < inputs; ++j) {
            int src = 0;
            while (slot_of[src] != j) ++src;
            if (!check(cudaMemcpyAsync(in_ptr(sl, src), static_cast<const char*>(srcs[src]) + off, n,
                                       cudaMemcpyHostToDevice, hp->in),
                       "host-to-device copy"))
                return VRWKV_ERR_CUDA;
        }
        if (!check(cudaEventRecord(hp->loaded[sl], hp->in), "event record") ||
            !check(cudaStreamWaitEvent(s, hp->loaded[sl], 0), "stream wait"))
            return VRWKV_ERR_CUDA;
        const vrwkv_status st = fused_entry(true, in_ptr(sl, 2), in_ptr(sl, 0), in_ptr(sl, 1), w, u, out_ptr(sl),
                                            nb, T, C, dtype, qs, s);
        if (st != VRWKV_OK) return st;
        if (!check(cudaEventRecord(hp->done[sl], s), "event record") ||
            !check(cudaStreamWaitEvent(hp->outs, hp->done[sl], 0), "stream wait") ||
            !check(cudaMemcpyAsync(static_cast<char*>(out) + off, out_ptr(sl), n, cudaMemcpyDeviceToHost,
                                   hp->outs),
                   "device-to-host copy") ||
            !check(cudaEventRecord(hp->freed[sl], hp->outs), "event record"))
            return VRWKV_ERR_CUDA;
    }
    // the caller's stream completes after the last copy back
    if (!check(cudaEventRecord(hp->freed[0], hp->outs), "event record") ||
        !check(cudaStreamWaitEvent(s, hp->freed[0], 0), "stream wait"))
        return VRWKV_ERR_CUDA;
    return ok();
}

}  // namespace

extern "C" {

vrwkv_status shift_entry(const void* x, void* out, const float* mu, int B, int H, int W, int C,
                         int shift_pixel, double gamma, int ng, vrwkv_dtype dtype, void* stream) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || H <= 0 || W <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, H, W and C must be positive");
    if ((long long)H * W > 0x7fffffffLL) return fail(VRWKV_ERR_UNSUPPORTED, "H*W too large");
    if (shift_pixel < 0) return fail(VRWKV_ERR_INVALID_ARG, "shift_pixel must be >= 0");
    if (!(gamma >= 0.0 && gamma <= 0.25)) return fail(VRWKV_ERR_INVALID_ARG, "gamma must lie in [0, 1/4]");
    if (!x || !out) return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    const int es = elem_bytes(dtype);
    if (!aligned(x, es) || !aligned(out, es) || (mu && !aligned(mu, 4)))
        return fail(VRWKV_ERR_INVALID_ARG, "pointer misaligned");
    const long long T = (long long)H * W;
    const size_t nbytes = (size_t)B * T * C * es;
    if (overlaps(out, nbytes, x, nbytes)) return fail(VRWKV_ERR_INVALID_ARG, "output overlaps the input");
    if (mu && overlaps(out, nbytes, mu, (size_t)C * 4))
        return fail(VRWKV_ERR_INVALID_ARG, "output overlaps mu");

    QshiftParams p;
    p.x = static_cast<const char*>(x);
    p.out = static_cast<char*>(out);
    p.mu = mu;
    p.BT = (long long)B * T;
    p.T = (int)T;
    p.C = C;
    p.H = H;
    p.W = W;
    p.s = shift_pixel;
    p.g = qs_bounds(C, gamma);
    p.ng = ng;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    {
        vrwkv_status st = VRWKV_OK;
        void* outs[1] = {out};
        const float* mus[1] = {mu};
        if (launch_qs_mix<1>(x, outs, mus, B, H, W, C, shift_pixel, gamma, ng, dtype, s, &st)) return st;
    }
    const bool vec = ((size_t)C * es) % 16 == 0 && aligned(x, 16) && aligned(out, 16);
    const long long work = vec ? p.BT * (C / (16 / es)) : p.BT * C;
    const int threads = 256;
    const long long blocks = std::min<long long>((work + threads - 1) / threads, 148LL * 16);
    if (vec) {
        if (dtype == VRWKV_F32) qshift_vec_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(p);
        else qshift_vec_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(p);
    } else {
        if (dtype == VRWKV_F32) qshift_scalar_kernel<float><<<(unsigned)blocks, threads, 0, s>>>(p);
        else qshift_scalar_kernel<__nv_bfloat16><<<(unsigned)blocks, threads, 0, s>>>(p);
    }
    return cuda_status(cudaGetLastError(), "qshift kernel launch");
}

vrwkv_status vrwkv_qshift(const void* x, void* out, const float* mu, int B, int H, int W, int C,
                          int shift_pixel, double gamma, vrwkv_dtype dtype, void* stream) {
    return shift_entry(x, out, mu, B, H, W, C, shift_pixel, gamma, 4, dtype, stream);
}

vrwkv_status vrwkv_bishift(const void* x, void* out, const float* mu, int B, int H, int W, int C,
                           int shift_pixel, double gamma, vrwkv_dtype dtype, void* stream) {
    return shift_entry(x, out, mu, B, H, W, C, shift_pixel, gamma, 2, dtype, stream);
}

vrwkv_status vrwkv_channel_mix(const void* x, void* out, int B, int T, int C, vrwkv_dtype dtype,
                               const vrwkv_qshift_params* qs, void* stream) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!x || !out) return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    if ((long long)B * T > 0x7fffffffLL) return fail(VRWKV_ERR_UNSUPPORTED, "B*T must be below 2^31");
    const int es = elem_bytes(dtype);
    if (!aligned(x, es) || !aligned(out, es)) return fail(VRWKV_ERR_INVALID_ARG, "pointer misaligned");
    const size_t nbytes = (size_t)B * T * C * es;
    if (overlaps(out, nbytes, x, nbytes)) return fail(VRWKV_ERR_INVALID_ARG, "output overlaps the input");
    ChannelMixParams p;
    p.x = static_cast<const char*>(x);
    p.out = static_cast<char*>(out);
    p.mu_r = p.mu_k = nullptr;
    p.BT = B * T;
    p.T = T;
    p.C = C;
    p.H = 1;
    p.W = T;
    p.s = 0;
    p.g = no_shift_bounds();  // without qs every channel reads its own token: QS is the identity
    p.ng = 4;
    if (qs) {
        vrwkv_status st = check_qs(qs, T, C);
        if (st != VRWKV_OK) return st;
        p.mu_r = qs->mu_r;
        p.mu_k = qs->mu_k;
        p.H = qs->H;
        p.W = qs->W;
        p.s = qs->shift_pixel;
        p.g = qs_bounds(C, qs->gamma);
        p.ng = shifted_groups(qs);
        for (const float* m : {p.mu_r, p.mu_k})
            if (m && overlaps(out, nbytes, m, (size_t)C * 4))
                return fail(VRWKV_ERR_INVALID_ARG, "output overlaps mu");
    }
    p.divT = make_fastdiv((unsigned)p.T);
    p.divW = make_fastdiv((unsigned)p.W);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nv = 16 / es;  // channels per 16-byte vector
    const bool vec = (C % nv) == 0 && bounds_multiple_of(p.g, nv) && aligned(x, 16) && aligned(out, 16) &&
                     (!p.mu_r || aligned(p.mu_r, 8)) && (!p.mu_k || aligned(p.mu_k, 8));
    if (!vec) {
        const long long n = (long long)p.BT * C;
        const long long blocks = std::min<long long>((n + 255) / 256, 148LL * 16);
        if (dtype == VRWKV_F32) channel_mix_scalar_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(p);
        else channel_mix_scalar_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(p);
        g_last_kernel = "channel_mix_scalar_kernel";
        return cuda_status(cudaGetLastError(), "channel_mix kernel launch");
    }
    p.UR = C / nv;
    static std::atomic<int> occ[2] = {{0}, {0}};
    dim3 grid, block;
    const int di = dtype == VRWKV_F32 ? 0 : 1;
    vrwkv_status st = dtype == VRWKV_F32
        ? column_launch(channel_mix_vec_kernel<float>, occ[di], p.UR, p.BT, &grid, &block)
        : column_launch(channel_mix_vec_kernel<__nv_bfloat16>, occ[di], p.UR, p.BT, &grid, &block);
    if (st != VRWKV_OK) return st;
    if (dtype == VRWKV_F32) channel_mix_vec_kernel<float><<<grid, block, 0, s>>>(p);
    else channel_mix_vec_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(p);
    g_last_kernel = "channel_mix_vec_kernel";
    return cuda_status(cudaGetLastError(), "channel_mix kernel launch");
}

size_t vrwkv_block_workspace_bytes(int B, int T, int C, vrwkv_dtype dtype) {
    if (B <= 0 || T <= 0 || C <= 0 || (dtype != VRWKV_F32 && dtype != VRWKV_BF16)) return 0;
    return 6 * block_ws_slot(B, T, C, dtype) + 4 * block_wt_slot(C, dtype);
}

vrwkv_status vrwkv_spatial_mix_block(const void* x, const void* w_r, const void* w_k, const void* w_v,
                                     const void* w_o, const float* w, const float* u, const float* ln_gamma,
                                     const float* ln_beta, float ln_eps, void* out, int B, int T, int C,
                                     vrwkv_dtype dtype, const vrwkv_qshift_params* qs, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!x || !w_r || !w_k || !w_v || !w_o || !w || !u || !ln_gamma || !ln_beta || !out || !qs || !workspace)
        return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    if (!(ln_eps >= 0.0f)) return fail(VRWKV_ERR_INVALID_ARG, "ln_eps must be >= 0");
    if ((long long)B * T > 0x7fffffffLL) return fail(VRWKV_ERR_UNSUPPORTED, "B*T must be below 2^31");
    {
        vrwkv_status st = check_qs(qs, T, C);
        if (st != VRWKV_OK) return st;
    }
    const void* mats[6] = {x, w_r, w_k, w_v, w_o, out};
    for (const void* m : mats)
        if (!aligned(m, 16)) return fail(VRWKV_ERR_INVALID_ARG, "token and weight tensors must be 16-byte aligned");
    const float* vecs[4] = {w, u, ln_gamma, ln_beta};
    for (const float* f : vecs)
        if (!aligned(f, 4)) return fail(VRWKV_ERR_INVALID_ARG, "float32 vector misaligned");
    if (!aligned(workspace, 256)) return fail(VRWKV_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const size_t need = vrwkv_block_workspace_bytes(B, T, C, dtype);
    if (workspace_bytes < need)
        return fail(VRWKV_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu needed",
                    workspace_bytes, need);
    const int es = elem_bytes(dtype);
    const size_t nb = (size_t)B * T * C * es, wb = (size_t)C * C * es;
    struct Span { const void* p; size_t n; };
    const Span ins[11] = {{x, nb}, {w_r, wb}, {w_k, wb}, {w_v, wb}, {w_o, wb}, {w, (size_t)C * 4},
                          {u, (size_t)C * 4}, {ln_gamma, (size_t)C * 4}, {ln_beta, (size_t)C * 4},
                          {qs->mu_r, (size_t)C * 4}, {qs->mu_k, (size_t)C * 4}};
    for (const Span& in : ins) {
        if (overlaps(out, nb, in.p, in.n)) return fail(VRWKV_ERR_INVALID_ARG, "output overlaps an input");
        if (overlaps(workspace, need, in.p, in.n))
            return fail(VRWKV_ERR_INVALID_ARG, "workspace overlaps an input");
    }
    if (overlaps(workspace, need, out, nb) || overlaps(workspace, need, qs->mu_v, (size_t)C * 4) ||
        overlaps(out, nb, qs->mu_v, (size_t)C * 4))
        return fail(VRWKV_ERR_INVALID_ARG, "workspace or output overlaps");

    // the three Q-Shift mixes (one pass over x when the vector kernel
    // applies, else three), then the three projections
    const size_t slot = block_ws_slot(B, T, C, dtype);
    char* base = static_cast<char*>(workspace);
    void* sh[3] = {base, base + slot, base + 2 * slot};
    void* bR = base + 3 * slot;
    void* bK = base + 4 * slot;
    void* bV = base + 5 * slot;
    char* wts_t = base + 6 * slot;  // transposed weights (bfloat16 GEMM operands)
    const size_t wslot = block_wt_slot(C, dtype);
    void* t0 = sh[0];
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int M = B * T;
    const float* mus[3] = {qs->mu_r, qs->mu_k, qs->mu_v};
    const void* wts[3] = {w_r, w_k, w_v};
    void* dst[3] = {bR, bK, bV};
    vrwkv_status qst = VRWKV_OK;
    bool wo_ready = false;  // W_O already transposed (with the other three)
    // bfloat16: the mixes as the projections' A-operand producer (one fused
    // launch, nothing staged in HBM) where the shape allows
    const bool fused = dtype == VRWKV_BF16 && block_fused_wanted() && !gemm_single_cta_forced() &&
                       gemm_qs_project(x, wts, mus, dst, B, T, C, qs, wts_t, wslot, s, &qst);
    if (fused && qst != VRWKV_OK) return qst;
    if (!fused) {
        const bool walked = mus[0] && mus[1] && mus[2] &&
                            launch_qs_mix<3>(x, sh, mus, B, qs->H, qs->W, C, qs->shift_pixel, qs->gamma,
                                             shifted_groups(qs), dtype, s, &qst);
        if (walked && qst != VRWKV_OK) return qst;
        if (!walked) {
            for (int i = 0; i < 3; ++i) {
                vrwkv_status st = shift_entry(x, sh[i], mus[i], B, qs->H, qs->W, C, qs->shift_pixel,
                                              qs->gamma, shifted_groups(qs), dtype, stream);
                if (st != VRWKV_OK) return st;
            }
        }
        // the four weights transposed in one launch where it applies
        const void* w4[4] = {w_r, w_k, w_v, w_o};
        void* wt4[4] = {wts_t, wts_t + wslot, wts_t + 2 * wslot, wts_t + 3 * wslot};
        wo_ready = dtype == VRWKV_BF16 && launch_transpose_pairs(w4, wt4, 4, C, C, s);
        for (int i = 0; i < 3; ++i) {
            vrwkv_status st = gemm_project(sh[i], wts[i], dst[i], M, C, C, dtype, wts_t + i * wslot, s, wo_ready);
            if (st != VRWKV_OK) return st;
        }
    }
    // sigma(R) (.) Bi-WKV(K, V) on the projected channels (Q-Shift already
    // applied before the projections), into t0
    vrwkv_status st = vrwkv_spatial_gate(bR, bK, bV, w, u, t0, B, T, C, dtype, nullptr, stream);
    if (st != VRWKV_OK) return st;
    // W_O into the R buffer (dead after the gate), then LayerNorm into out
    st = gemm_project(t0, w_o, bR, M, C, C, dtype, wts_t + 3 * wslot, s, wo_ready);
    if (st != VRWKV_OK) return st;
    LayerNormParams lp;
    lp.x = static_cast<const char*>(bR);
    lp.y = static_cast<char*>(out);
    lp.g = ln_gamma;
    lp.b = ln_beta;
    lp.rows = M;
    lp.C = C;
    lp.eps = ln_eps;
    lp.vec = ((size_t)C * es) % 16 == 0;
    const unsigned blocks = (unsigned)((M + 7) / 8);
    // 16-byte vectors per lane of the register-resident kernel (0: three-pass)
    const int vpl = (lp.vec && aligned(ln_gamma, 16) && aligned(ln_beta, 16))
                        ? (int)(((size_t)C * es / 16 + 31) / 32) : 0;
    auto launch_ln = [&](auto io) {
        using IO = decltype(io);
        if (vpl >= 1 && vpl <= 1) layer_norm_reg_kernel<IO, 1><<<blocks, 256, 0, s>>>(lp);
        else if (vpl == 2) layer_norm_reg_kernel<IO, 2><<<blocks, 256, 0, s>>>(lp);
        else if (vpl >= 3 && vpl <= 4) layer_norm_reg_kernel<IO, 4><<<blocks, 256, 0, s>>>(lp);
        else if (vpl >= 5 && vpl <= 8) layer_norm_reg_kernel<IO, 8><<<blocks, 256, 0, s>>>(lp);
        else layer_norm_kernel<IO><<<blocks, 256, 0, s>>>(lp);
    };
    if (dtype == VRWKV_F32) launch_ln(float{});
    else launch_ln(__nv_bfloat16{});
    st = cuda_status(cudaGetLastError(), "layer_norm_kernel launch");
    if (st == VRWKV_OK) g_last_kernel = "spatial_mix_block";
    return st;
}

vrwkv_status vrwkv_spatial_gate_static(const void* r, const void* k, const void* v, const float* w,
                                       const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
                                       const vrwkv_qshift_params* qs, void* stream) {
    // the argument checks that need no device come first, so an invalid call
    // leaves the device untouched (the launch path repeats them all)
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!r || !k || !v || !w || !u || !out) return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    if (qs) {
        vrwkv_status st = check_qs(qs, T, C);
        if (st != VRWKV_OK) return st;
    }
    const WsLayout L = ws_layout(B, C);
    if (L.bytes > kStaticWsBytes)
        return fail(VRWKV_ERR_UNSUPPORTED,
                    "B*ceil(C/8) = %lld columns need %zu bytes of exchange state; the static workspace "
                    "holds %zu",
                    (long long)B * ((C + fast::kCS - 1) / fast::kCS), L.bytes, kStaticWsBytes);
    const WsLayout LW = wide_ws_layout(B, T, C);
    if (T > kWideSegTokens && LW.bytes > kStaticWsBytes)
        return fail(VRWKV_ERR_UNSUPPORTED,
                    "B*C/16*ceil(T/4096) = %lld column segments need %zu bytes of exchange state; the static "
                    "workspace holds %zu",
                    (long long)B * (C / wide::kCW) * ((T + kWideSegTokens - 1) / kWideSegTokens), LW.bytes,
                    kStaticWsBytes);
    unsigned char* ws = static_workspace();
    if (!ws) return fail(VRWKV_ERR_CUDA, "cannot locate the static workspace");
    // counters and flags start at zero for every call (a previous call that
    // stopped on an error may have left them set); the records need no reset
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(ws, 0, std::max(L.recs_off, LW.recs_off), s);
    if (e != cudaSuccess) return cuda_status(e, "clearing the static workspace");
    return fused_entry(true, r, k, v, w, u, out, B, T, C, dtype, qs, stream, true, ws, kStaticWsBytes);
}

vrwkv_status vrwkv_biwkv_bwd(const void* k, const void* v, const float* w, const float* u,
                             const void* gy, void* gk, void* gv, float* gw, float* gu, float* gw_total,
                             float* gu_total, int B, int T, int C, vrwkv_dtype dtype, void* stream) {
    if (dtype != VRWKV_F32 && dtype != VRWKV_BF16)
        return fail(VRWKV_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B <= 0 || T <= 0 || C <= 0)
        return fail(VRWKV_ERR_INVALID_ARG, "B, T and C must be positive (got %d, %d, %d)", B, T, C);
    if (!k || !v || !w || !u || !gy || !gk || !gv || !gw || !gu)
        return fail(VRWKV_ERR_INVALID_ARG, "required pointer is NULL");
    if (T > bwd::kMaxT) return fail(VRWKV_ERR_UNSUPPORTED, "T = %d exceeds %d", T, bwd::kMaxT);
    const int es = elem_bytes(dtype);
    const void* toks[5] = {k, v, gy, gk, gv};
    for (const void* t : toks)
        if (!aligned(t, es)) return fail(VRWKV_ERR_INVALID_ARG, "token tensor misaligned");
    const float* vecs[6] = {w, u, gw, gu, gw_total, gu_total};
    for (const float* f : vecs)
        if (f && !aligned(f, 4)) return fail(VRWKV_ERR_INVALID_ARG, "float32 vector misaligned");
    const size_t nb = (size_t)B * T * C * es, nbc = (size_t)B * C * 4, nc = (size_t)C * 4;
    struct Span { const void* p; size_t n; };
    const Span ins[5] = {{k, nb}, {v, nb}, {gy, nb}, {w, nc}, {u, nc}};
    const Span outs[6] = {{gk, nb}, {gv, nb}, {gw, nbc}, {gu, nbc}, {gw_total, nc}, {gu_total, nc}};
    for (int i = 0; i < 6; ++i) {
        for (const Span& in : ins)
            if (overlaps(outs[i].p, outs[i].n, in.p, in.n))
                return fail(VRWKV_ERR_INVALID_ARG, "an output overlaps an input");
        for (int j2 = i + 1; j2 < 6; ++j2)
            if (overlaps(outs[i].p, outs[i].n, outs[j2].p, outs[j2].n))
                return fail(VRWKV_ERR_INVALID_ARG, "outputs overlap");
    }
    bwd::Params p;
    p.imaj = 0;
    p.k = static_cast<const char*>(k);
    p.v = static_cast<const char*>(v);
    p.g = static_cast<const char*>(gy);
    p.w = w;
    p.u = u;
    p.gk = static_cast<char*>(gk);
    p.gv = static_cast<char*>(gv);
    p.gw = gw;
    p.gu = gu;
    p.B = B;
    p.T = T;
    p.C = C;
    p.Tc = std::min(T, bwd::kTc);
    p.ncl = (T + p.Tc - 1) / p.Tc;
    p.invT = (float)(1.0 / (double)T);
    p.vec = (C % 2 == 0);
    for (const void* t : toks) p.vec = p.vec && aligned(t, 2 * es);
    // k, v and gy by TMA (tiles of 8 channels x 512 tokens as two boxes of 256
    // strided tokens, element stride 8 along T, as the forward kernel's) when
    // the shape and alignment allow
    p.tma = 0;
    p.tma_store = 0;
    p.err = device_error_word();
    if (!tma_disabled() && C % bwd::kCS == 0 && p.err && aligned(k, 16) && aligned(v, 16) && aligned(gy, 16)) {
        EncodeTiledFn enc = encode_fn();
        if (enc) {
            const void* srcs[3] = {k, v, gy};
            const CUtensorMapDataType tdt =
                dtype == VRWKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
            const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
            const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)T * C * es};
            const cuuint32_t box[3] = {(cuuint32_t)bwd::kCS, 256u, 1};  // 32 strided rows
            const cuuint32_t estr[3] = {1, (cuuint32_t)bwd::kL, 1};
            bool okm = true;
            for (int i = 0; i < 3 && okm; ++i)
                okm = enc(&p.map[i], tdt, 3, const_cast<void*>(srcs[i]), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
            p.tma = okm ? 1 : 0;
            // optionally, gk, gv leave by TMA stores in the same layout (a CTA
            // spans 512 tokens or ends the column, so no box reaches another
            // CTA's tokens)
            void* dsts[2] = {gk, gv};
            bool oks = okm && aligned(gk, 16) && aligned(gv, 16) && bwd_tma_store_enabled();
            for (int i = 0; i < 2 && oks; ++i)
                oks = enc(&p.omap[i], tdt, 3, dsts[i], dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
            p.tma_store = oks ? 1 : 0;
        }
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the 16-token tensor-memory kernel where the inputs arrive by TMA and gk,
    // gv can leave by TMA stores
    if (p.tma && !bwd_tm_disabled() && aligned(gk, 16) && aligned(gv, 16)) {
        bwd::Params p2 = p;
        EncodeTiledFn enc = encode_fn();
        const CUtensorMapDataType tdt =
            dtype == VRWKV_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        const cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
        const cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)T * C * es};
        const cuuint32_t box[3] = {(cuuint32_t)bwd::kCS, 256u, 1};
        const cuuint32_t estr[3] = {1, (cuuint32_t)bwd::kL, 1};
        void* dsts[2] = {gk, gv};
        bool oks = enc != nullptr;
        // residue-major views (tokens as (C, T / 8, 8, B), one box per 512-token
        // tile) where T is a multiple of 8: a CTA's boxes are then one load per
        // input and one store per output instead of sixteen each
        p2.imaj = 0;
        if (oks && T % 8 == 0 && !tm_imaj_disabled()) {
            const void* srcs[3] = {k, v, gy};
            const cuuint64_t rdims[4] = {(cuuint64_t)C, (cuuint64_t)T / 8, 8, (cuuint64_t)B};
            const cuuint64_t rstrides[3] = {(cuuint64_t)8 * C * es, (cuuint64_t)C * es, (cuuint64_t)T * C * es};
            const cuuint32_t rbox[4] = {(cuuint32_t)bwd::kCS, (cuuint32_t)(bwd2::kTc / 8), 8, 1};
            const cuuint32_t restr[4] = {1, 1, 1, 1};
            bool okr = true;
            for (int i = 0; i < 3 && okr; ++i)
                okr = enc(&p2.map[i], tdt, 4, const_cast<void*>(srcs[i]), rdims, rstrides, rbox, restr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
            for (int i = 0; i < 2 && okr; ++i)
                okr = enc(&p2.omap[i], tdt, 4, dsts[i], rdims, rstrides, rbox, restr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
            if (okr) {
                p2.imaj = 1;
            } else {
                p2.map[0] = p.map[0];
                p2.map[1] = p.map[1];
                p2.map[2] = p.map[2];
            }
        }
        for (int i = 0; i < 2 && oks && !p2.imaj; ++i)
            oks = enc(&p2.omap[i], tdt, 3, dsts[i], dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                      CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        if (oks) {
            bool fell_back = false;
            vrwkv_status st = dtype == VRWKV_F32 ? launch_bwd_tm<float>(p2, s, &fell_back)
                                                 : launch_bwd_tm<__nv_bfloat16>(p2, s, &fell_back);
            if (st != VRWKV_OK) return st;
            if (!fell_back) {
                const int blocks = (C + 255) / 256;
                if (gw_total) bwd::batch_sum_kernel<<<blocks, 256, 0, s>>>(gw, gw_total, B, C);
                if (gu_total) bwd::batch_sum_kernel<<<blocks, 256, 0, s>>>(gu, gu_total, B, C);
                return cuda_status(cudaGetLastError(), "batch_sum_kernel launch");
            }
        }
    }
    auto kern = dtype == VRWKV_F32 ? bwd::biwkv_bwd_kernel<float> : bwd::biwkv_bwd_kernel<__nv_bfloat16>;
    {
        static std::atomic<int> granted[2] = {{0}, {0}};
        cudaError_t e = ensure_smem(kern, granted[dtype == VRWKV_F32 ? 0 : 1], (int)bwd::kSmemBytes);
        if (e != cudaSuccess) return cuda_status(e, "cudaFuncSetAttribute");
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.ncl, (C + bwd::kCS - 1) / bwd::kCS, B);
    cfg.blockDim = dim3(bwd::kThreads, 1, 1);
    cfg.dynamicSmemBytes = bwd::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.ncl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
    attr[1].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicyLoadBalancing;
    cfg.attrs = attr;
    cfg.numAttrs = p.ncl > 1 ? 2 : 0;
    if (p.ncl > 1) {
        // clusters of at most 8 CTAs (T <= 4096): a portable size
        static_assert(bwd::kClusterMax <= 8, "portable cluster size");
        static std::atomic<int> checked[2][bwd::kClusterMax + 1];
        const int di = dtype == VRWKV_F32 ? 0 : 1;
        cudaError_t e;
        int v2 = checked[di][p.ncl].load();
        if (v2 == 0) {
            int n = 0;
            e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
            v2 = (e == cudaSuccess && n > 0) ? 1 : -1;
            if (e != cudaSuccess) cudaGetLastError();
            checked[di][p.ncl].store(v2);
        }
        if (v2 < 0)
            return fail(VRWKV_ERR_UNSUPPORTED, "a cluster of %d backward CTAs cannot be scheduled", p.ncl);
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return cuda_status(e, "biwkv_bwd_kernel launch");
    g_last_kernel = "biwkv_bwd_kernel";
    const int blocks = (C + 255) / 256;
    if (gw_total) bwd::batch_sum_kernel<<<blocks, 256, 0, s>>>(gw, gw_total, B, C);
    if (gu_total) bwd::batch_sum_kernel<<<blocks, 256, 0, s>>>(gu, gu_total, B, C);
    return cuda_status(cudaGetLastError(), "batch_sum_kernel launch");
}

vrwkv_status vrwkv_biwkv_fwd(const void* k, const void* v, const float* w, const float* u, void* wkv,
                             int B, int T, int C, vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
                             void* stream) {
    return fused_entry(false, nullptr, k, v, w, u, wkv, B, T, C, dtype, qs, stream);
}

vrwkv_status vrwkv_spatial_gate(const void* r, const void* k, const void* v, const float* w,
                                const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
                                const vrwkv_qshift_params* qs, void* stream) {
    return fused_entry(true, r, k, v, w, u, out, B, T, C, dtype, qs, stream);
}

size_t vrwkv_spatial_gate_host_buffer_bytes(int slice_b, int T, int C, vrwkv_dtype dtype, int inputs) {
    if (slice_b <= 0 || T <= 0 || C <= 0 || inputs < 1 || inputs > 3 ||
        (dtype != VRWKV_F32 && dtype != VRWKV_BF16))
        return 0;
    return kHostSlots * host_slot_bytes(slice_b, T, C, elem_bytes(dtype), inputs);
}

vrwkv_status vrwkv_spatial_gate_host(const void* r, const void* k, const void* v, const float* w,
                                     const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
                                     const vrwkv_qshift_params* qs, int slice_b, void* dev_buf,
                                     size_t dev_buf_bytes, void* stream) {
    return host_pipeline(r, k, v, w, u, out, B, T, C, dtype, qs, slice_b, dev_buf, dev_buf_bytes,
                         static_cast<cudaStream_t>(stream));
}

size_t vrwkv_fwd_workspace_bytes(int B, int T, int C) {
    if (B <= 0 || T <= 0 || C <= 0) return 0;
    return std::max(ws_layout(B, C).bytes, wide_ws_layout(B, T, C).bytes);
}

vrwkv_status vrwkv_biwkv_fwd_ws(const void* k, const void* v, const float* w, const float* u, void* wkv,
                                int B, int T, int C, vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
                                void* workspace, size_t workspace_bytes, void* stream) {
    return fused_entry(false, nullptr, k, v, w, u, wkv, B, T, C, dtype, qs, stream, true, workspace,
                       workspace_bytes);
}

vrwkv_status vrwkv_spatial_gate_ws(const void* r, const void* k, const void* v, const float* w,
                                   const float* u, void* out, int B, int T, int C, vrwkv_dtype dtype,
                                   const vrwkv_qshift_params* qs, void* workspace, size_t workspace_bytes,
                                   void* stream) {
    return fused_entry(true, r, k, v, w, u, out, B, T, C, dtype, qs, stream, true, workspace,
                       workspace_bytes);
}

const char* vrwkv_status_string(vrwkv_status status) {
    switch (status) {
    case VRWKV_OK: return "VRWKV_OK";
    case VRWKV_ERR_INVALID_ARG: return "VRWKV_ERR_INVALID_ARG";
    case VRWKV_ERR_UNSUPPORTED: return "VRWKV_ERR_UNSUPPORTED";
    case VRWKV_ERR_CUDA: return "VRWKV_ERR_CUDA";
    case VRWKV_ERR_TIMEOUT: return "VRWKV_ERR_TIMEOUT";
    default: return "VRWKV_ERR_UNKNOWN";
    }
}

const char* vrwkv_last_error(void) { return g_last_error.c_str(); }

const char* vrwkv_last_kernel(void) { return g_last_kernel; }

vrwkv_status vrwkv_set_wait_limit(double seconds) {
    if (!(seconds > 0.0 && seconds <= 60.0))
        return fail(VRWKV_ERR_INVALID_ARG, "wait limit must lie in (0, 60] seconds");
    const unsigned long long ns = (unsigned long long)(seconds * 1e9);
    return cuda_status(cudaMemcpyToSymbol(fast::g_vrwkv_wait_ns, &ns, sizeof(ns)), "setting the wait limit");
}

vrwkv_status vrwkv_device_status(void) {
    unsigned int* word = device_error_word();
    if (!word) return fail(VRWKV_ERR_CUDA, "cannot locate the device error word");
    unsigned int v = 0;
    cudaError_t e = cudaMemcpy(&v, word, sizeof(v), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e, "reading the device error word");
    if (v == 0) return ok();
    const unsigned int zero = 0;
    e = cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e, "clearing the device error word");
    return fail(VRWKV_ERR_TIMEOUT,
                "kernel-side failure (flags 0x%x: 1 = TMA tile wait ran out, 2 = wait for a column "
                "peer's record ran out, 4 = workspace not zero-filled)",
                v);
}

}  // extern "C"
