/*
 * vrwkv.h -- C ABI of the B200 (sm_100a) Vision-RWKV spatial-mix core.
 *
 * The operations follow "OpenGVLab&港中文&复旦&南大&清华提出Vision-RWKV
 * Backbone" (cloud.tencent.com article 2395249) and the q_shift listing on
 * "LinXin's Blog" (Vision-RWKV entry):
 *   - Q-Shift, Quad-Directional Token Shift, eq. 9;
 *   - Bi-WKV, Linear Complexity Bidirectional Attention, eq. 5
 *     (equivalently the RNN form, eq. 6-7);
 *   - the receptance gate sigma(R) (.) wkv, Overall Architecture, eq. 2;
 *   - the channel-mix gate sigma(R_c) (.) SquaredReLU(K_c), Overall
 *     Architecture, eq. 3-4;
 *   - the spatial-mix block with its projections and LayerNorm, eq. 1-2;
 *   - the Bi-WKV backward pass: the pages state that one exists (in an
 *     appendix they do not reproduce), so vrwkv_biwkv_bwd computes the plain
 *     derivatives of eq. 5.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  Token tensors are dense row-major (B, T, C): channel fastest, then
 *   token, then batch.  With a patch grid H x W the token index is
 *   t = h*W + w (raster order) and T = H*W.  w, u and the mu vectors are
 *   dense float32 vectors of length C.
 * Memory.  Every pointer is caller-owned DEVICE memory, except the token
 *   buffers of vrwkv_spatial_gate_host (page-locked host memory).  No call
 *   allocates device memory; vrwkv_spatial_gate_host creates two copy
 *   streams and a few events once per device.  The only device memory the
 *   library owns is
 *   reserved when it loads: a device error word and the fixed workspace of
 *   vrwkv_spatial_gate_static.
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream).  Work is enqueued asynchronously; the caller
 *   synchronises.  vrwkv_spatial_gate (and its _ws variant),
 *   vrwkv_channel_mix, vrwkv_spatial_mix_block and vrwkv_biwkv_bwd enqueue
 *   kernel launches only and are replayed from CUDA graphs by the benchmark;
 *   capture of the other calls has not been tested.
 * Dtypes.  VRWKV_F32 or VRWKV_BF16 select the storage type of the token
 *   tensors (inputs and output alike).  Arithmetic is float32 throughout;
 *   bfloat16 outputs are rounded to nearest even once, at the store.
 * Aliasing.  Inputs may alias one another (the spatial-mix core commonly
 *   passes one tensor x as r, k and v).  An output must not overlap any
 *   input: that is VRWKV_ERR_INVALID_ARG.
 * Errors.  Every entry point validates its arguments on the host before it
 *   touches the GPU and returns a status; nothing aborts and no exception
 *   crosses the ABI.  vrwkv_last_error() gives a one-line reason for the most
 *   recent non-OK status of the calling thread.  VRWKV_ERR_CUDA reports a
 *   launch failure (the CUDA error string is in vrwkv_last_error()); errors of
 *   kernels that already ran asynchronously surface at the caller's next
 *   synchronisation, as usual in CUDA.
 */
#ifndef VRWKV_H
#define VRWKV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VRWKV_OK = 0,
    VRWKV_ERR_INVALID_ARG = 1, /* bad size, pointer, alignment or parameter */
    VRWKV_ERR_UNSUPPORTED = 2, /* valid problem outside the kernels' limits */
    VRWKV_ERR_CUDA = 3,        /* the CUDA runtime reported an error        */
    VRWKV_ERR_TIMEOUT = 4      /* a kernel's bounded wait ran out (see
                                  vrwkv_device_status)                      */
} vrwkv_status;

typedef enum {
    VRWKV_F32 = 0,
    VRWKV_BF16 = 1
} vrwkv_dtype;

/*
 * Q-Shift parameters (eq. 9 and the q_shift listing).
 *   H, W         patch grid; T must equal H*W.
 *   shift_pixel  shift distance in patches, >= 0.  A distance at or beyond
 *                the grid extent leaves that channel group all zero.
 *   gamma        channel-group fraction, 0 <= gamma <= 1/4.  The groups end
 *                at the listing's slice bounds b_j = int(C*gamma*j), j = 1..4,
 *                evaluated as Python does (C*gamma in double, then times j,
 *                then truncated).  Channels [0,b_1) take x[h, w-s], [b_1,b_2)
 *                x[h, w+s], [b_2,b_3) x[h-s, w], [b_3,b_4) x[h+s, w] (zero
 *                outside the grid); channels >= b_4 take x[h, w] unchanged
 *                (none at gamma = 1/4, where the bounds are eq. 9's C/4, C/2,
 *                3C/4, C).  Groups differ in size when C*gamma is not an
 *                integer: C = 10, gamma = 1/4 gives [0,2) [2,5) [5,7) [7,10).
 *   mu_r, mu_k, mu_v  device float32[C] interpolation weights, each nullable.
 *                With mu the shifted input is mu*x + (1-mu)*x_shift; a NULL
 *                mu means the shifted tensor x_shift itself.
 *   mode         VRWKV_QSHIFT_QUAD, or VRWKV_QSHIFT_BIDIR for sparse inputs:
 *                the pages pre-train with MAE after turning Q-Shift into a
 *                bidirectional shift and say no more; this mode keeps the two
 *                row groups ([0,b_1) from x[h, w-s], [b_1,b_2) from x[h, w+s],
 *                zero past the row) and passes every other channel through.  A
 *                sparse input is one row of its visible tokens (H = 1).
 */
typedef enum {
    VRWKV_QSHIFT_QUAD = 0,  /* Q-Shift, eq. 9: four shifted channel groups   */
    VRWKV_QSHIFT_BIDIR = 1  /* bidirectional shift for sparse (MAE) inputs: */
                            /* the two row groups only                      */
} vrwkv_qshift_mode;

typedef struct {
    int H;
    int W;
    int shift_pixel;
    double gamma;
    const float* mu_r;
    const float* mu_k;
    const float* mu_v;
    int mode;  /* vrwkv_qshift_mode */
} vrwkv_qshift_params;

/*
 * vrwkv_qshift -- Q-Shift of one tensor (eq. 9; q_shift listing).
 *   x    (B, H*W, C) input, dtype `dtype`.
 *   out  (B, H*W, C) output, same dtype, must not overlap x.
 *   mu   float32[C] or NULL: out = x_shift (NULL) or mu*x + (1-mu)*x_shift,
 *        evaluated in float32 as t1 = mu*x, t2 = (1-mu)*x_shift, t1 + t2 with
 *        each operation rounded separately (no fused multiply-add), then
 *        stored (rounded to bfloat16 for VRWKV_BF16).  Without mu the result
 *        is a pure gather and bit-exact in either dtype.
 * Errors: INVALID_ARG for B, H, W or C <= 0, shift_pixel < 0, gamma outside
 *   [0, 1/4], NULL x/out, misaligned pointers, or out overlapping x.
 */
vrwkv_status vrwkv_qshift(const void* x, void* out, const float* mu, int B,
                          int H, int W, int C, int shift_pixel, double gamma,
                          vrwkv_dtype dtype, void* stream);

/*
 * vrwkv_bishift -- the VRWKV_QSHIFT_BIDIR shift of one tensor (see
 * vrwkv_qshift_params.mode); arguments, mix, exactness and errors as
 * vrwkv_qshift.
 */
vrwkv_status vrwkv_bishift(const void* x, void* out, const float* mu, int B,
                           int H, int W, int C, int shift_pixel, double gamma,
                           vrwkv_dtype dtype, void* stream);

/*
 * vrwkv_biwkv_fwd -- Bi-WKV forward (eq. 5):
 *   wkv_t = [ sum_{i!=t} e^{-(|t-i|-1)/T * w + k_i} v_i + e^{u + k_t} v_t ]
 *         / [ sum_{i!=t} e^{-(|t-i|-1)/T * w + k_i}     + e^{u + k_t}     ]
 * independently for every batch b and channel c, with w[c] of either sign.
 *   k, v  (B, T, C) inputs, dtype `dtype`.
 *   w, u  float32[C] decay and current-token bonus.
 *   wkv   (B, T, C) output, same dtype, must not overlap k, v, w or u.
 *   qs    NULL, or Q-Shift parameters applied to k (mu_k) and v (mu_v) on
 *         load (mu_r is ignored); T must then equal qs->H * qs->W.
 * Kernels (the same results up to rounding):
 *   - the 32-token tensor-memory kernel, the default for T > 512: the
 *     8-channel kernel's conditions with 1024-token CTAs, T <= 8192, and
 *     the thread-block cluster and tensor memory of four CTAs per SM
 *     available; each thread's per-token partial sums are kept in tensor
 *     memory between its two passes.  Where T is a multiple of 8 a tile
 *     arrives in one TMA box and the results leave in one;
 *   - the 8-channel TMA kernel, the default up to 512 tokens (256-token
 *     CTAs for T <= 256): C % 8 == 0, 16-byte-aligned inputs and, with qs,
 *     group bounds int(C*gamma*j) that are multiples of 8, T <= 8192.
 *     Q-Shift reads the image (C, W, H, B) where W % 8 == 0, W <= 256 and
 *     whole image rows make whole warps, else the flat tokens with the
 *     shifted tiles displaced by the group's token offset (row-wrapped
 *     tokens cleared after the load);
 *   - the 16-channel slab kernel, with VRWKV_FORWARD=wide in the
 *     environment (and for long sequences through the workspace variants):
 *     C % 16 == 0, T % 16 == 0, T <= 4096, 16-byte-aligned tensors and,
 *     with qs, bounds that are multiples of 16, W % 16 == 0, shift_pixel 1
 *     where a horizontal group exists and shift_pixel*W <= 256 for the
 *     vertical ones;
 *   - a generic kernel for everything else (T <= 4096).
 *   Setting VRWKV_DISABLE_TMA=1 in the environment forces the generic
 *   kernel, VRWKV_FORWARD=tm takes the tensor-memory kernel at any T where it
 *   qualifies and VRWKV_FORWARD=narrow never, VRWKV_TM_ROT=0 keeps its
 *   sub-chunks in natural order, VRWKV_TM_IMAJ=0 and VRWKV_TM_OSTORE=0 keep
 *   its loads and stores on lane-strided boxes, VRWKV_QS_VIEW=flat (image)
 *   takes Q-Shift through the flat token view wherever it can (never),
 *   VRWKV_SHORT_CTA=0 keeps short columns on 512-token CTAs,
 *   VRWKV_DISABLE_WIDE=1 keeps the 16-channel one off, VRWKV_TMA_CHUNK=8
 *   holds the 8-channel kernel to 8-token thread chunks and
 *   VRWKV_NO_TMA_STORE=1 to per-thread stores of its results (diagnostics).
 * Limits: T <= 8192 on the 8-channel kernel, 4096 on the others
 *   (UNSUPPORTED above; the workspace variants below reach 32768); on the
 *   generic kernel with qs, a halo of shift_pixel*W tokens must fit its
 *   shared-memory tile.
 *   Exponents are renormalised by the running maximum of k, so a constant
 *   added to every k of a channel leaves wkv unchanged; results stay finite
 *   while |w| + (spread of k within a channel) stays well below 80.
 * Errors: INVALID_ARG for B, T or C <= 0, NULL k/v/w/u/wkv, misaligned
 *   pointers, an overlapping output, or bad qs fields (see the struct).
 */
vrwkv_status vrwkv_biwkv_fwd(const void* k, const void* v, const float* w,
                             const float* u, void* wkv, int B, int T, int C,
                             vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
                             void* stream);

/*
 * vrwkv_spatial_gate -- the spatial-mix core without projections (eq. 2
 * with identity W_R, W_K, W_V and no W_O):
 *   out = sigma(QS_R(r)) (.) Bi-WKV(QS_K(k), QS_V(v)),  sigma(z) = 1/(1+e^{-z})
 * where QS_* is Q-Shift with mu_r, mu_k, mu_v when qs is given and the
 * identity when qs is NULL.  r, k and v may be the same tensor (eq. 1 shifts
 * one X three ways); that case reads the tensor once.
 *   r, k, v  (B, T, C) inputs, dtype `dtype`.
 *   w, u     float32[C].
 *   out      (B, T, C) output, same dtype, must not overlap any input.
 * Limits and errors as vrwkv_biwkv_fwd, with r also required non-NULL.
 */
vrwkv_status vrwkv_spatial_gate(const void* r, const void* k, const void* v,
                                const float* w, const float* u, void* out,
                                int B, int T, int C, vrwkv_dtype dtype,
                                const vrwkv_qshift_params* qs, void* stream);

/*
 * vrwkv_spatial_gate_host -- vrwkv_spatial_gate on HOST buffers, for callers
 * whose tokens live in host memory: the same operation (eq. 2, eq. 5, eq. 9),
 * with the host <-> device traffic overlapped with the computation.  The
 * batch is cut into slices of slice_b rows (each (b, c) column is
 * independent and Q-Shift mixes tokens of one batch row only, so a slice is
 * an exact sub-problem); slice i is copied host -> device into slot i % n of
 * dev_buf (n = 3 slots, or 2 when dev_buf holds only two) on a library copy
 * stream, computed on `stream`, and copied back on a second copy stream, so
 * both copy directions and the kernels overlap.
 * Results equal vrwkv_spatial_gate's bit for bit.
 *   r, k, v   (B, T, C) inputs in page-locked host memory (cudaHostAlloc or
 *             cudaHostRegister); they may be the same buffer, copied once.
 *   w, u      float32[C] in device memory; qs as for vrwkv_spatial_gate (its
 *             mu vectors in device memory).
 *   out       (B, T, C) page-locked host output, must not overlap an input.
 *   slice_b   batch rows per slice, 1 <= slice_b <= B.
 *   dev_buf   caller-owned device staging, 256-byte aligned, of at least
 *             vrwkv_spatial_gate_host_buffer_bytes(slice_b, T, C, dtype,
 *             number of distinct input buffers) bytes.
 * Asynchronous on `stream`: work already queued there runs first, and the
 * stream (so a synchronisation on it) completes after the last copy back;
 * the host buffers must stay valid until then.  The library creates its two
 * copy streams and a few events once per device and keeps them; calls from
 * several host threads are serialised while they enqueue.
 * Errors: INVALID_ARG for bad sizes, NULL pointers, an out-of-range slice_b,
 *   a small or misaligned dev_buf, pageable host memory or an overlapping
 *   output; the rest as vrwkv_spatial_gate.
 */
vrwkv_status vrwkv_spatial_gate_host(const void* r, const void* k,
                                     const void* v, const float* w,
                                     const float* u, void* out, int B, int T,
                                     int C, vrwkv_dtype dtype,
                                     const vrwkv_qshift_params* qs,
                                     int slice_b, void* dev_buf,
                                     size_t dev_buf_bytes, void* stream);

/* Device staging bytes vrwkv_spatial_gate_host uses for slices of slice_b
 * batch rows with `inputs` (1 to 3) distinct input buffers (three slots; two
 * thirds of it is the minimum it accepts); 0 for invalid arguments. */
size_t vrwkv_spatial_gate_host_buffer_bytes(int slice_b, int T, int C,
                                            vrwkv_dtype dtype, int inputs);

/*
 * Workspace variants of vrwkv_biwkv_fwd and vrwkv_spatial_gate.  Same
 * operations, arguments and results.  Up to 4096 tokens, the CTAs of one
 * (b, 8-channel) column exchange their partial sums through the caller's
 * workspace instead of a thread-block cluster, which frees the kernel from
 * cluster co-scheduling (the 32-token tensor-memory kernel above 512 tokens,
 * the 8-channel kernel up to 512).  Longer sequences (up to T = 32768, e.g. the
 * 16384 tokens of a 2048^2 image at patch 16) run on the 16-channel kernel
 * when the shape qualifies for it: a column splits into segments of one
 * 8-CTA cluster (4096 tokens); segments take tickets from a counter in the
 * workspace, publish their totals there and wait, bounded, for the other
 * segments of their column.
 *   workspace        device memory of at least vrwkv_fwd_workspace_bytes(B,
 *                    T, C) bytes, 256-byte aligned, owned by the caller.  It
 *                    must be zero-filled once before its first use; the
 *                    kernels leave it ready for the next call (counters reset,
 *                    a generation number advanced).  Calls that may run at
 *                    the same time (other streams) need separate workspaces;
 *                    calls queued on one stream may share one.
 *   workspace_bytes  its size.
 * The CTAs of a column wait for one another with a bounded spin (the wait
 * limit, 2 s by default; see vrwkv_set_wait_limit); a
 * timeout is recorded in the device error word (see vrwkv_device_status).
 * Errors: as the plain entry points, plus INVALID_ARG for a NULL, misaligned,
 *   too small or overlapping workspace.
 */
size_t vrwkv_fwd_workspace_bytes(int B, int T, int C);

vrwkv_status vrwkv_biwkv_fwd_ws(const void* k, const void* v, const float* w,
                                const float* u, void* wkv, int B, int T, int C,
                                vrwkv_dtype dtype,
                                const vrwkv_qshift_params* qs, void* workspace,
                                size_t workspace_bytes, void* stream);

vrwkv_status vrwkv_spatial_gate_ws(const void* r, const void* k, const void* v,
                                   const float* w, const float* u, void* out,
                                   int B, int T, int C, vrwkv_dtype dtype,
                                   const vrwkv_qshift_params* qs,
                                   void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * vrwkv_spatial_gate_static -- vrwkv_spatial_gate_ws on a workspace the
 * library owns, for callers that cannot allocate device memory (a fixed
 * memory budget, an allocator they may not call at this point): the call
 * allocates nothing.  The pages have no counterpart of this entry point; it
 * exists only for such callers.
 * The workspace is one 4 MiB array per device, reserved when the library is
 * loaded, which holds the exchange state of B * ceil(C / 8) <= ~1600 columns;
 * larger problems return VRWKV_ERR_UNSUPPORTED.  Each call first clears the
 * array's counters and flags on `stream` (cudaMemsetAsync), then runs the
 * workspace kernel; results equal vrwkv_spatial_gate's.
 * Calls that overlap in time (other streams, other host threads) share the
 * one array and race: serialise them, or use vrwkv_spatial_gate_ws with a
 * workspace per stream.
 * Arguments, results, limits and errors otherwise as vrwkv_spatial_gate.
 */
vrwkv_status vrwkv_spatial_gate_static(const void* r, const void* k,
                                       const void* v, const float* w,
                                       const float* u, void* out, int B, int T,
                                       int C, vrwkv_dtype dtype,
                                       const vrwkv_qshift_params* qs,
                                       void* stream);

/*
 * vrwkv_spatial_mix_block -- the spatial-mix block with its projections
 * (Overall Architecture, eq. 1-2, with Q-Shift of eq. 9 and Bi-WKV of eq. 5):
 *   R = QS_R(x) W_R,  K = QS_K(x) W_K,  V = QS_V(x) W_V             (eq. 1)
 *   O = (sigma(R) (.) Bi-WKV(K, V)) W_O                              (eq. 2)
 *   out = LayerNorm(O) = ln_gamma * (O - mean) / sqrt(var + ln_eps) + ln_beta
 * (LayerNorm over channels, biased variance; the pages normalise after the
 * output projection).  Residual connections are left to the caller.
 *   x          (B, T, C) input, dtype `dtype`, 16-byte aligned.
 *   w_r, w_k, w_v, w_o  (C, C) weights, dtype `dtype`, row-major (C_in,
 *              C_out): a token row times the matrix; 16-byte aligned.
 *   w, u       float32[C] Bi-WKV decay and bonus of the projected channels.
 *   ln_gamma, ln_beta  float32[C]; ln_eps >= 0.
 *   out        (B, T, C) output, dtype `dtype`, 16-byte aligned.
 *   qs         required: grid, shift, gamma and mu_r, mu_k, mu_v.
 *   workspace  device memory of at least vrwkv_block_workspace_bytes(B, T,
 *              C, dtype) bytes, 256-byte aligned: six (B, T, C) staging
 *              buffers and the four weights transposed to (C_out, C_in).
 * Steps (all on `stream`): the three Q-Shift mixes (one pass over x; each
 * bit-identical to vrwkv_qshift's), three projection GEMMs, the fused
 * vrwkv_spatial_gate core on the projected R, K, V, the W_O GEMM and a
 * LayerNorm kernel.  The GEMMs are the library's own: for bfloat16 a
 * tcgen05 tensor-core kernel (TMA tiles with the 128-byte swizzle, float32
 * accumulators in tensor memory, results rounded to bfloat16 once; CTA
 * pairs with cta_group::2 MMAs, or single CTAs with VRWKV_GEMM_1CTA=1) after
 * a transpose of each weight into the workspace; for float32 a kernel on the
 * FP32 pipes.  bfloat16 needs C % 8 == 0.  The sigma(R) gate is applied in
 * the core's epilogue, so W_O reads the gated result directly.
 * VRWKV_BLOCK_FUSED=1 projects R, K, V in one launch whose A operand is the
 * Q-Shift mix made in shared memory from x and its shifted copy (no staging
 * in HBM; bit-identical to the staged path) where bfloat16, C a multiple of
 * 256 up to 1024, T % 128 == 0, W dividing 128 (or a multiple of it) and
 * group bounds that are multiples of 64 allow; off by default (slower on the
 * B200, 521 against 424 us at B = 8, 64 x 64, C = 1024: it mixes each x tile
 * once per output tile).
 * Errors: INVALID_ARG for bad sizes, NULL or misaligned pointers, overlaps,
 *   bad qs fields or a small workspace; UNSUPPORTED for B*T >= 2^31, a
 *   bfloat16 C that is not a multiple of 8, or the core's limits; CUDA for a
 *   failed launch.  A GEMM wait that runs out sets flag 8 of the device
 *   error word (vrwkv_device_status).
 */
size_t vrwkv_block_workspace_bytes(int B, int T, int C, vrwkv_dtype dtype);

vrwkv_status vrwkv_spatial_mix_block(const void* x, const void* w_r,
                                     const void* w_k, const void* w_v,
                                     const void* w_o, const float* w,
                                     const float* u, const float* ln_gamma,
                                     const float* ln_beta, float ln_eps,
                                     void* out, int B, int T, int C,
                                     vrwkv_dtype dtype,
                                     const vrwkv_qshift_params* qs,
                                     void* workspace, size_t workspace_bytes,
                                     void* stream);

/*
 * vrwkv_biwkv_bwd -- gradients of Bi-WKV (eq. 5) for an upstream gradient gy
 * = dL/dwkv, by the chain rule.  For each (b, c) column, with
 * W_ti = e^{-(|t-i|-1)/T * w} (i != t), W_tt = e^u, D_t = sum_i W_ti e^{k_i}
 * and wkv_t the forward output:
 *   gk_i = e^{k_i} sum_t W_ti gy_t (v_i - wkv_t) / D_t
 *   gv_i = e^{k_i} sum_t W_ti gy_t / D_t
 *   gu   = sum_t e^{u + k_t} gy_t (v_t - wkv_t) / D_t
 *   gw   = -(1/T) sum_t sum_{i != t} (|t-i|-1) W_ti e^{k_i} gy_t (v_i - wkv_t) / D_t
 * The forward sums are recomputed from k, v, w, u (nothing is saved from the
 * forward call).
 *   k, v, gy  (B, T, C) inputs, dtype `dtype`.
 *   w, u      float32[C].
 *   gk, gv    (B, T, C) outputs, dtype `dtype` (rounded once for VRWKV_BF16).
 *   gw, gu    float32[B*C] outputs: row b holds batch element b's share; the
 *             gradient of the shared w and u is their sum over b.
 *   gw_total, gu_total  float32[C] or NULL: if given, that sum over b, taken
 *             in order b = 0..B-1 by a second kernel on the same stream.
 * Arithmetic is float32; dw and du are summed in a fixed order, so repeated
 * calls give identical bits.  With C % 8 == 0 and 16-byte-aligned k, v, gy
 * the inputs arrive by TMA, else by direct loads (VRWKV_DISABLE_TMA=1 forces
 * the direct loads; same results).  With TMA inputs and 16-byte-aligned gk,
 * gv the default kernel gives each thread 16 tokens and keeps its per-token
 * states in tensor memory (VRWKV_BWD_TM=0: the 8-token kernel; the same
 * results up to rounding); on the 8-token kernel VRWKV_BWD_TMA_STORE=1 also
 * stores gk, gv by TMA from shared memory (same results; measured slower,
 * hence off by default).
 * Limits: T <= 4096 (UNSUPPORTED above, or when the GPU cannot co-schedule
 *   the thread-block cluster a column needs); the exponent range is that of
 *   vrwkv_biwkv_fwd.
 * Errors: INVALID_ARG for B, T or C <= 0, NULL required pointers, misaligned
 *   pointers, or an output that overlaps an input or another output.
 */
vrwkv_status vrwkv_biwkv_bwd(const void* k, const void* v, const float* w,
                             const float* u, const void* gy, void* gk, void* gv,
                             float* gw, float* gu, float* gw_total,
                             float* gu_total, int B, int T, int C,
                             vrwkv_dtype dtype, void* stream);

/*
 * vrwkv_channel_mix -- the elementwise part of the channel-mix module (eq. 3-4
 * with identity W_R, W_K, W_V and no W_O):
 *   out = sigma(QS_R(x)) (.) SquaredReLU(QS_K(x)),  SquaredReLU(z) = max(z, 0)^2
 * where QS_R, QS_K are Q-Shift with qs->mu_r and qs->mu_k (qs->mu_v is
 * ignored), or the identity when qs is NULL.
 *   x    (B, T, C) input, dtype `dtype`.
 *   out  (B, T, C) output, same dtype, must not overlap x, mu_r or mu_k.
 *   qs   NULL, or Q-Shift parameters; T must then equal qs->H * qs->W.
 * Arithmetic: float32, with the mix evaluated as x_shift + mu*(x - x_shift)
 *   (fused multiply-add) and sigma(r) = 1/(1 + 2^(-r*log2 e)) from the hardware
 *   exp2 and reciprocal; one rounding to bfloat16 at the store for VRWKV_BF16.
 * Kernels: a vector kernel serves C*sizeof(dtype) % 16 == 0 with 16-byte-
 *   aligned x and out, 8-byte-aligned mu and group bounds int(C*gamma*j) that
 *   are multiples of 16/sizeof(dtype); everything else runs a scalar kernel.
 * Errors: INVALID_ARG for B, T or C <= 0, NULL x/out, misaligned pointers, an
 *   overlapping output or bad qs fields; UNSUPPORTED for B*T >= 2^31.
 */
vrwkv_status vrwkv_channel_mix(const void* x, void* out, int B, int T, int C,
                               vrwkv_dtype dtype, const vrwkv_qshift_params* qs,
                               void* stream);

/*
 * vrwkv_device_status -- report and clear kernel-side failures on the
 * current device.  Kernels that wait for their asynchronous (TMA) tile
 * copies (bit 0) or, in the workspace variants, for the records of the other
 * CTAs of a column (bit 1) give up after the wait limit (two seconds unless
 * vrwkv_set_wait_limit changes it); a workspace
 * variant that finds its workspace in an invalid state (not zero-filled
 * before first use; bit 2) stops at once.  Each records the failure in a
 * device error word and finishes (its outputs are then undefined) instead
 * of hanging.  This call synchronises with the current device, reads that
 * word, clears it and returns VRWKV_ERR_TIMEOUT if it was set, VRWKV_OK
 * otherwise (VRWKV_ERR_CUDA if the device cannot be read); the bits are in
 * vrwkv_last_error().
 */
vrwkv_status vrwkv_device_status(void);

/*
 * vrwkv_set_wait_limit -- how long every bounded wait in the library's
 * kernels (TMA tile completion, a cluster peer's mailbox record, a column
 * peer's workspace record) may last before it gives up, records its bit in
 * the device error word and lets the kernel finish.  The pages have no
 * counterpart: this bounds the damage of a lost peer or copy.
 *   seconds  0 < seconds <= 60 (default 2), measured on the GPU's global
 *            timer.
 * Applies to the current device, for every later launch on it.  It is a
 * synchronous copy into device memory: call it outside stream capture and
 * while no kernel of this library runs on the device.  A limit far below
 * the kernels' normal run time makes healthy launches report timeouts.
 * Errors: INVALID_ARG for a limit outside (0, 60]; VRWKV_ERR_CUDA if the
 * device cannot be written.
 */
vrwkv_status vrwkv_set_wait_limit(double seconds);

/* Name of the main kernel the calling thread's most recent successful
 * vrwkv_biwkv_fwd / vrwkv_spatial_gate / vrwkv_channel_mix / vrwkv_biwkv_bwd
 * call launched ("" before any), e.g. "biwkv_tma_kernel",
 * "biwkv_fused_kernel", "channel_mix_vec_kernel" or "biwkv_bwd_kernel".
 * Diagnostics only. */
const char* vrwkv_last_kernel(void);

/* Static, never-NULL name of a status code. */
const char* vrwkv_status_string(vrwkv_status status);

/* One-line reason for the calling thread's most recent non-OK status
 * ("" if none).  Valid until that thread's next call into the library. */
const char* vrwkv_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* VRWKV_H */
