/*
 * svdq.h -- C ABI of libsvdq, the SVDQuant W4A4 linear layer with its 16-bit
 * low-rank branch, for NVIDIA B200 (sm_100a).
 *
 *     Y = (X diag(lambda)^-1) L1 L2  +  Q4(X diag(lambda)^-1) Q4(R),
 *     R = diag(lambda) W - L1 L2.
 *
 * What the layer computes is described in "Nunchaku Lite: the 50% VRAM
 * reduction now integrated into Diffusers" (axbrief.com), section "The
 * Mechanics of 4-Bit Efficiency and SVDQuant": activation outliers are moved
 * into the weights, the weight is split into a 16-bit low-rank branch and a
 * 4-bit residual, and the residual branch runs with 4-bit weights and 4-bit
 * activations (W4A4).  The two-call structure (down projection inside the
 * activation quantiser, up projection inside the 4-bit GEMM, both sharing the
 * activations) follows "Problemas do Nunchaku Qwen e como corrigi-los em
 * 2025" (apatero.com), section "O que e Nunchaku e como acelera modelos Qwen".
 * The capability gate follows the Nunchaku Lite article, section "Hardware
 * Specialization and the Compression Workflow".
 *
 * Conventions for every call:
 *   - Pointers named *_host are host memory; every other data pointer is
 *     device memory owned by the caller, unless stated otherwise.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy stream).
 *   - Work is enqueued asynchronously on `stream`; the return value reports
 *     host-side validation and launch errors only.  Device-side failures
 *     (a bounded wait that timed out) are recorded in the handle and
 *     reported by svdq_device_status().
 *   - There is no CPU fallback: on a machine without an sm_100 GPU every
 *     compute call returns SVDQ_ERR_UNSUPPORTED_DEVICE or SVDQ_ERR_CUDA.
 *   - A handle must not be used on two streams at the same time.
 *
 * Shapes: M tokens, K in-features, N out-features, r rank.
 *   K % 128 == 0, N % 16 == 0, r in {0, 16, 32, 64, 128}, 1 <= M <= max_M.
 *   Rows beyond M inside the last 128-row tile are never written.
 *
 * Formats (all row-major, K contiguous):
 *   bf16 values are passed as their 16-bit patterns (uint16_t).
 *   4-bit codes: two per byte, element 2j in the low nibble.
 *     INT4 : two's complement -8..7, group G = 64 along K, bf16 scales.
 *     NVFP4: E2M1 (sign bit 3, magnitude index 0..7 = 0,0.5,1,1.5,2,3,4,6),
 *            group G = 16 along K, E4M3 scale bytes.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad flag */
  SVDQ_ERR_SHAPE = 2,              /* M/K/N/r outside the supported set */
  SVDQ_ERR_ALIGNMENT = 3,          /* a device pointer is not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 4, /* no CUDA device, or not compute capability 10.x */
  SVDQ_ERR_OOM = 5,                /* device allocation failed */
  SVDQ_ERR_CUDA = 6,               /* any other CUDA runtime / driver error */
  SVDQ_ERR_DEVICE_TIMEOUT = 7,     /* a kernel's bounded wait expired */
  SVDQ_ERR_RANGE = 8               /* a value outside the range the selected path
                                      computes exactly (see SVDQ_INT4_F16) */
} svdq_status;

typedef enum {
  SVDQ_INT4_G64_BF16 = 0,   /* INT4 codes, group 64, bf16 scales */
  SVDQ_NVFP4_G16_E4M3 = 1   /* E2M1 codes, group 16, E4M3 scales */
} svdq_variant;

/* svdq_weight_desc.flags */
#define SVDQ_EPI_GELU 1u    /* apply GELU (tanh form) in the GEMM epilogue */
/* NVFP4 only: run kernel 2 on single SMs (128 x 256 tiles) for every M.  By
 * default, when M > 128, it runs on pairs of SMs: a two-CTA cluster per
 * 256 x 256 tile, one M = 256 tensor-core MMA stream per pair, which halves
 * the B bytes each SM stages and so deepens the pipeline (B200, fc1
 * 4608 x 3072 x 12288: 108.5 vs 118.8 us side by side).  Both compute the same y up to
 * fp32 summation order.  For comparison and tests. */
#define SVDQ_GEMM_SINGLE_SM 2u
/* INT4 only: run kernel 2 as one fp16 GEMM of the dequantised operands
 * (s_x q_x) and (s_w q_w) on the 16-bit tensor cores (kind::f16) instead of
 * per-group int8 MMAs with an fp32 rescale of every group.  Both operands are
 * exact in fp16 -- a bf16 scale has 8 significant bits, |q| <= 8 at most 3 --
 * while the scales stay in fp16's range, and every product is exact in the
 * fp32 accumulator, so y equals the int8 path's up to fp32 summation order.
 * svdq_weights_load returns SVDQ_ERR_RANGE if a dequantised weight is not an
 * fp16 value; svdq_device_status returns SVDQ_ERR_RANGE after a call in
 * which an activation scale exceeded 9357 (7 s > 65504).  Activation scales
 * below 2^-17 lose low bits of s q (absolute error below 2^-25 s). */
#define SVDQ_INT4_F16 4u
/* NVFP4 only, not with SVDQ_EPI_GELU: the layer is a merged QKV projection
 * whose N = 3 H 128 output columns are [Q | K | V] (heads of 128 features);
 * the GEMM epilogue RMS-normalises every head of Q and of K,
 *   v <- v / sqrt(mean_head(v^2) + norm_eps) * g   (g = q_norm or k_norm),
 * and rotates its interleaved pairs (2i, 2i+1) by the token's rotary angle
 * for pair i: (a, b) <- (a cos - b sin, a sin + b cos).  V is stored as is.
 * Defined by "Nunchaku Lite ..." (axbrief.com), section "The Trade-off
 * Between Fused Kernels and Generality": QKV projection, Q/K normalisation
 * and rotary embeddings bundled into one kernel over a merged to_qkv module.
 * Such a layer runs through svdq_linear_forward_qkv /
 * svdq_w4a4_gemm_lowrank_up_qkv only.  N % 384 == 0. */
#define SVDQ_EPI_QKV_NORM_ROPE 8u

typedef struct svdq_weights* svdq_weights_t;   /* opaque, library-owned */

/*
 * Pre-packed layer weights, all HOST memory, read only during
 * svdq_weights_load (the library copies what it needs).
 *   lambda   fp32 [K]        smoothing factors (> 0); the library stores
 *                            fp32(1 / lambda) for the runtime multiply
 *   L1       bf16 [K x r]    low-rank down factor
 *   L2       bf16 [r x N]    low-rank up factor
 *   w_codes  u8   [N x K/2]  residual codes, one row per output feature
 *   w_scales INT4: bf16 [N x K/64]; NVFP4: E4M3 bytes [N x K/16]
 *   bias     bf16 [N] or NULL
 *   w_scale_exp  NVFP4 only: per-tensor second-level scale 2^w_scale_exp of
 *            the residual weights (a weight is code * E4M3 scale *
 *            2^w_scale_exp); 0 = none.  |w_scale_exp| <= 100, else
 *            SVDQ_ERR_INVALID_ARG (also for INT4 with a nonzero value).
 *            The GEMM multiplies its accumulator by 2^e and T by 2^-e, both
 *            exact, so y is the same function of the dequantised weights.
 * L1 / L2 may be NULL when r == 0.
 */
typedef struct {
  svdq_variant variant;
  int64_t K, N, r, max_M;
  uint32_t flags;
  const float* lambda;
  const uint16_t* L1;
  const uint16_t* L2;
  const uint8_t* w_codes;
  const void* w_scales;
  const uint16_t* bias;
  int32_t w_scale_exp;
  /* SVDQ_EPI_QKV_NORM_ROPE only (else ignored): host bf16 [128] RMS-norm
   * weights of the Q and K heads and the epsilon (0 < norm_eps < 1) */
  const uint16_t* q_norm;
  const uint16_t* k_norm;
  float norm_eps;
} svdq_weight_desc;

/*
 * Defined by: "Nunchaku Lite ..." (axbrief.com), section "The Mechanics of
 * 4-Bit Efficiency and SVDQuant" -- the layer's weights are the smoothing
 * (outliers shifted from activations into weights), a 16-bit low-rank branch
 * and a 4-bit residual; section "Hardware Specialization and the Compression
 * Workflow" -- INT4 or NVFP4 precision, a CUDA capability check that refuses
 * unsupported devices; "Nunchaku 1.3.0 ..." (note.com), section "SVDQ-FP4 on
 * Blackwell", item "1. INT4" -- INT4 codes are -8..+7 times a scale.
 * Copy and re-tile the weights into library-owned device memory on the
 * current device and size the forward workspace for max_M tokens.
 * The weight scales of the NVFP4 variant are re-tiled into the tensor-core
 * scale-factor layout; the INT4 residual codes are additionally kept as int8
 * for the int8 tensor-core path (with SVDQ_INT4_F16: as fp16 s_w q_w
 * [N x K] instead, SVDQ_ERR_RANGE if a value is not exact in fp16).  On error
 * *out is left NULL and nothing is allocated.
 */
svdq_status svdq_weights_load(const svdq_weight_desc* desc, svdq_weights_t* out, void* stream);

/* Free a handle (NULL is a no-op).  Synchronises the device first.  No
 * counterpart on the pages: resource release for svdq_weights_load. */
svdq_status svdq_weights_free(svdq_weights_t h);

/*
 * Layout helper for kernel 1's output (no counterpart on the pages).
 * Size in bytes of the activation-scale buffer for M tokens:
 *   INT4 : M * (K/64) * 2          canonical [M x K/64] bf16
 *   NVFP4: ceil(M/128)*128 * (K/16) the tensor-core tiled layout (below)
 */
svdq_status svdq_act_scales_bytes(svdq_weights_t h, int64_t M, size_t* bytes);

/*
 * Defined by: "Problemas do Nunchaku Qwen ..." (apatero.com), section "O que
 * e Nunchaku e como acelera modelos Qwen" -- the low-rank down projection is
 * fused with the activation quantisation kernel so both branches share the
 * activations; "Nunchaku Lite ..." (axbrief.com), section "The Mechanics of
 * 4-Bit Efficiency and SVDQuant" -- activation outliers are divided out
 * before the activations are quantised to 4 bits (W4A4).
 * Kernel 1: smooth, quantise and pack the activations, and compute the
 * rank-r down projection from the same tiles.
 *   x          bf16 [M x K]
 *   act_codes  u8   [M x K/2]  (written)
 *   act_scales see svdq_act_scales_bytes (written).  NVFP4 layout: 128-row
 *              tiles; inside tile b, K-block j (64 elements = 4 scales) of
 *              row m sits at byte
 *                b*(K/64)*512 + j*512 + (m%32)*16 + ((m/32)%4)*4 + (k/16)%4
 *   t          fp32 [M x r]  T = X' L1 (written; untouched when r == 0).
 *              When a row block's K range is split over several CTAs (M
 *              below about 74 * 128 tokens) the partial sums are added into
 *              t with fp32 reductions (the kernel clears t first), so
 *              its last bits (and through it Y's) may differ between calls
 *              on the same input -- unless svdq_set_deterministic is on.
 * Per element (round to nearest even throughout):
 *   x' = bf16(fp32(x) * inv_lambda);  a = max|x'| over the group;
 *   INT4 s = bf16(a / 7), q = rint(x'/s);  NVFP4 s = e4m3_satfinite(a / 6),
 *   q = e2m1_satfinite(x'/s);  s == 0 gives q = +0.  Codes are those of
 *   IEEE correctly rounded fp32 division x'/s.
 */
svdq_status svdq_quantize_act_lowrank_down(svdq_weights_t h, const void* x, int64_t M,
                                           uint8_t* act_codes, void* act_scales, float* t,
                                           void* stream);

/*
 * Defined by: "Problemas do Nunchaku Qwen ..." (apatero.com), section "O que
 * e Nunchaku e como acelera modelos Qwen" -- the up projection is fused with
 * the 4-bit compute kernel; "Nunchaku Lite ..." (axbrief.com), section "The
 * Mechanics of 4-Bit Efficiency and SVDQuant" -- the 4-bit residual branch
 * with 4-bit weights and activations, added to the 16-bit low-rank branch.
 * Kernel 2: the 4-bit GEMM on the packed residual with the low-rank up
 * projection, optional bias and GELU fused into the epilogue.
 *   act_codes, act_scales, t  as written by kernel 1 (t ignored when r == 0)
 *   y  bf16 [M x N]  (written)
 *   y = GELU?( sum_g s_x s_w sum_{k in g} q_x q_w  +  T L2  +  bias ),
 *   accumulated in fp32, rounded once to bf16.
 */
svdq_status svdq_w4a4_gemm_lowrank_up(svdq_weights_t h, const uint8_t* act_codes,
                                      const void* act_scales, const float* t, int64_t M,
                                      void* y, void* stream);

/*
 * Defined by: "Nunchaku Lite ..." (axbrief.com), section "The Mechanics of
 * 4-Bit Efficiency and SVDQuant" -- the quantised layer replaces a standard
 * linear layer (SVDQW4A4Linear in place of nn.Linear): y = layer(x).
 * Both kernels back to back through the handle's workspace.  Kernel 2 is
 * launched as a programmatic dependent of kernel 1 (its set-up overlaps
 * kernel 1's tail); every kernel of the library waits for the previous
 * kernel of the stream before it touches global memory.
 *   x  bf16 [M x K], y  bf16 [M x N]
 */
svdq_status svdq_linear_forward(svdq_weights_t h, const void* x, void* y, int64_t M,
                                void* stream);

/*
 * Defined by: the fused path of "Nunchaku Lite ..." (axbrief.com), section
 * "The Trade-off Between Fused Kernels and Generality" (see
 * SVDQ_EPI_QKV_NORM_ROPE).  Kernel 2 / the whole layer for a handle loaded
 * with SVDQ_EPI_QKV_NORM_ROPE:
 *   rope  device fp32 [M x 64 x 2], 16-byte aligned: (cos, sin) of the
 *         rotary angle of token m for pair i at rope[(m * 64 + i) * 2]
 * Other arguments as svdq_w4a4_gemm_lowrank_up / svdq_linear_forward.  The
 * GEMM is preceded by one small kernel that copies the table, row-blocked
 * (32 tokens per block, so that the epilogue's loads are contiguous), into
 * a buffer the handle owns (cdiv(max_M, 256) * 256 * 512 bytes, allocated at
 * load); the caller's table is read by that kernel and must stay valid until
 * it has run.  Calls on one handle from different streams at once race on
 * that buffer as on the workspace.
 */
svdq_status svdq_w4a4_gemm_lowrank_up_qkv(svdq_weights_t h, const uint8_t* act_codes,
                                          const void* act_scales, const float* t, int64_t M,
                                          const float* rope, void* y, void* stream);
svdq_status svdq_linear_forward_qkv(svdq_weights_t h, const void* x, const float* rope, void* y,
                                    int64_t M, void* stream);

/*
 * Defined by: "Problemas do Nunchaku Qwen ..." (apatero.com), section "O que
 * e Nunchaku e como acelera modelos Qwen" -- the down projection fused with
 * the quantisation kernel, the up projection with the 4-bit kernel, the
 * branches sharing the activations; "Nunchaku Lite ..." (axbrief.com),
 * section "The Trade-off Between Fused Kernels and Generality" -- fused
 * paths bundle operations to cut memory traffic.  Here two consecutive
 * layers (a DiT MLP's fc1 and fc2) share a kernel: fc1's GEMM epilogue
 * computes fc1's output y1 = bf16(GELU?(acc + bias)), then fc2's activation
 * side from it -- x2 = bf16(fp32(y1) * (1/lambda2)), fc2's NVFP4 codes and
 * scales (bit-identical to svdq_quantize_act_lowrank_down on y1) and
 * T2 = X2' L1_2 (tensor cores, fp32; several CTAs add into one row block
 * with fp32 atomics, so T2's summation order is not fixed) -- and y1 itself
 * is only stored when asked for.
 * Both handles NVFP4 (no QKV epilogue), h1's N == h2's K, N % 256 == 0,
 * h1's r in {0, 32}, h2's r in {16, 32}, else SVDQ_ERR_SHAPE / INVALID_ARG.
 *
 * svdq_w4a4_gemm_lowrank_up_chain: h1's kernel 2 on its activation codes,
 *   scales and T (as from svdq_quantize_act_lowrank_down on h1), writing
 *   h2's act_codes2 [M x N1/2], act_scales2 (tiled, svdq_act_scales_bytes of
 *   h2) and t2 fp32 [M x r2] (zeroed by the call on `stream`, then added
 *   into), and y1 bf16 [M x N1] unless y1 is NULL.
 * svdq_linear_forward_chain: y2 = fc2(fc1(x)) through the handles'
 *   workspaces: fc1's activation kernel, the fused kernel, fc2's GEMM.
 */
svdq_status svdq_w4a4_gemm_lowrank_up_chain(svdq_weights_t h1, const uint8_t* act_codes,
                                            const void* act_scales, const float* t, int64_t M, void* y1,
                                            svdq_weights_t h2, uint8_t* act_codes2, void* act_scales2,
                                            float* t2, void* stream);
svdq_status svdq_linear_forward_chain(svdq_weights_t h1, svdq_weights_t h2, const void* x, void* y2,
                                      int64_t M, void* stream);

/*
 * Defined by: the same layer as svdq_linear_forward.
 * Same as svdq_linear_forward with HOST input and output (pinned memory is
 * recommended; pageable memory works but its copies do not overlap): copies
 * x_host to the device, runs the layer and copies y back.  The rows go in
 * chunks (at least 256 rows, at most 8 chunks): a chunk's input copy and the
 * output copies of earlier chunks run on two streams of the handle while the
 * layer runs on `stream`, so the two copy directions and the kernels
 * overlap.  Y is the same as one svdq_linear_forward over all M rows (the
 * chunks use the activation kernel's K split of the whole M; with
 * svdq_set_deterministic, bit for bit).  Returns after enqueueing; `stream`
 * completes after the last output copy, so synchronise it before reading
 * y_host.  Device staging buffers, the two streams and their events are
 * owned by the handle (created on first use); calls on one handle must not
 * overlap.
 */
svdq_status svdq_linear_forward_host(svdq_weights_t h, const void* x_host, void* y_host,
                                     int64_t M, void* stream);

/*
 * Kernel 1 for callers that cannot allocate device memory: the same
 * smoothing, quantisation, packing and down projection as
 * svdq_quantize_act_lowrank_down, but with no weights handle and no call to
 * cudaMalloc or any other allocating routine, at load time or per call.
 * Code that runs inside a CUDA-graph capture, a runtime that owns every
 * device allocation (a fixed memory pool of an inference server, an
 * embedding plugin host), or a process with a hard device-memory budget
 * cannot let a library allocate; it passes every buffer itself:
 *   inv_lambda  device fp32 [K]      1 / lambda (the caller divides)
 *   l1t         device bf16 [r x K]  L1 transposed (NULL when r == 0)
 *   x, act_codes, act_scales, t      as for svdq_quantize_act_lowrank_down
 *   device_error device int, set to a nonzero wait-site code if a bounded
 *               wait expires (never cleared by the library).  May be NULL:
 *               such a failure is then reported to no one, and the outputs
 *               of that call may be incomplete without any sign of it
 * Unlike svdq_quantize_act_lowrank_down, T is summed over the K split in a
 * fixed order (bit-reproducible).  The split-K scratch (partial T tiles and
 * per-row-block arrival counters) lives in a static device array of the library: 10 MiB of partial tiles
 * plus counters for M <= 524288 tokens, held by every GPU that loads the
 * library until the process exits.  Calls whose split needs more, or with
 * M > 524288, return SVDQ_ERR_SHAPE before any work is enqueued.  The first
 * call on a device looks up the array's device address (once per device,
 * that device current); make that first call before any stream capture.
 * Every call shares the one array: the counters are cleared on `stream`
 * before each launch, and calls that overlap on the GPU (two streams, two
 * threads) race on it and must be serialised by the caller.
 * The method describes no counterpart to this entry point; it serves callers
 * that must not allocate.
 */
svdq_status svdq_quantize_act_lowrank_down_static(svdq_variant variant, int64_t K, int64_t r,
                                                  const float* inv_lambda, const uint16_t* l1t,
                                                  const void* x, int64_t M, uint8_t* act_codes,
                                                  void* act_scales, float* t, int* device_error,
                                                  void* stream);

/* ------------------------------------------------------------------------
 * AWQ W4A16 linear layer: 4-bit weights, 16-bit activations.
 *
 * Defined by: "Nunchaku Lite ..." (axbrief.com), section "The Mechanics of
 * 4-Bit Efficiency and SVDQuant" -- besides SVDQW4A4Linear the runtime
 * patching installs AWQW4A16Linear layers (4-bit weights, 16-bit
 * activations); section "The Trade-off Between Fused Kernels and
 * Generality" -- the scanner assigns AWQ W4A16 to modulation linear layers.
 * The pages give no arithmetic; the library computes (readings: activation-
 * aware channel factors a, groups of 64 along K, asymmetric unsigned codes
 * with an integer zero point):
 *   x' = fp32(x) * fp32(1/a_k)                       (kept in fp32)
 *   y[m,n] = sum_g s[n,g] sum_{k in g} x'[m,k] (q[n,k] - z[n,g])  (+ bias)
 * accumulated in fp32 and rounded once to bf16.  Modulation layers see one
 * token per image, so the call is a matrix-vector product bound by reading
 * the 4-bit weights; it runs on the CUDA cores.
 */
typedef struct svdq_awq* svdq_awq_t;   /* opaque, library-owned */

/* HOST memory, read only during svdq_awq_load:
 *   a       fp32 [K]        activation-aware channel factors (> 0)
 *   codes   u8   [N x K/2]  codes 0..15, element 2j in the low nibble
 *   scales  bf16 [N x K/64] group scales s
 *   zeros   u8   [N x K/64] integer zero points 0..15 (else INVALID_ARG)
 *   bias    bf16 [N] or NULL
 * Shapes: K % 64 == 0, 64 <= K <= 16384, 1 <= N, 1 <= M <= max_M. */
typedef struct {
  int64_t K, N, max_M;
  const float* a;
  const uint8_t* codes;
  const uint16_t* scales;
  const uint8_t* zeros;
  const uint16_t* bias;
} svdq_awq_desc;

/* Copy the weights into library-owned device memory on the current device
 * (1/a is computed once, by IEEE fp32 division).  On error *out is NULL. */
svdq_status svdq_awq_load(const svdq_awq_desc* desc, svdq_awq_t* out, void* stream);

/* Free a handle (NULL is a no-op).  Synchronises the device first. */
svdq_status svdq_awq_free(svdq_awq_t h);

/* y = layer(x): x bf16 [M x K] (4-byte aligned), y bf16 [M x N] (2-byte
 * aligned), device memory owned by the caller; asynchronous on `stream`,
 * launched as a programmatic dependent of the previous kernel (it waits for
 * that kernel before reading x). */
svdq_status svdq_awq_w4a16_forward(svdq_awq_t h, const void* x, void* y, int64_t M, void* stream);

/* ------------------------------------------------------------------------
 * Weight preparation on the GPU (offline compression; not on the layer's
 * timed path: these calls allocate scratch, copy small results to the host
 * and synchronise `stream` before returning).
 *
 * Defined by: "Nunchaku Lite ..." (axbrief.com), section "Hardware
 * Specialization and the Compression Workflow" -- inspect, calibrate the
 * data distribution to find outliers, quantize the weights, package, at INT4
 * or NVFP4 precision; section "The Mechanics of 4-Bit Efficiency and
 * SVDQuant" -- activation outliers shifted into the weights, the weights
 * split into a 16-bit low-rank branch and a 4-bit residual; "Problemas do
 * Nunchaku Qwen ..." (apatero.com), section "O que e Nunchaku ..." -- the
 * low-rank branch from a singular value decomposition.  The outputs are the
 * inputs of svdq_weights_load.  All pointers are device memory unless named
 * otherwise.
 */

/* Calibration and smoothing factors: lambda_k = max_m|x[m,k]|^alpha /
 * max_n|w[k,n]|^(1-alpha) (fp64, then fp32), 1 where either maximum is 0,
 * clamped to [2^-20, 2^20].  x bf16 [M x K] calibration activations, w bf16
 * [K x N] the layer's weight, lambda fp32 [K] (written). */
svdq_status svdq_prep_calibrate(const void* x, int64_t M, const void* w, int64_t K, int64_t N,
                                float alpha, float* lambda, void* stream);

/* Rank-r factors of W_hat = diag(lambda) w by a randomized SVD: the range
 * of W_hat Omega (omega fp32 [N x l], the caller's Gaussian test matrix,
 * r <= l <= 192, l <= min(K, N)) refined by `power_iters` power iterations
 * with re-orthonormalisation (Cholesky QR twice, fp64 Gram matrices), then
 * the small SVD of Q^T W_hat on the host in fp64.  The singular values are
 * split evenly: L1 = Q U_r S_r^(1/2) bf16 [K x r], L2 = S_r^(1/2) V_r^T bf16
 * [r x N] (round to nearest even).  The products with W_hat run in fp32. */
svdq_status svdq_prep_lowrank(const void* w, const float* lambda, int64_t K, int64_t N, int64_t r,
                              const float* omega, int64_t l, int power_iters, uint16_t* L1,
                              uint16_t* L2, void* stream);

/* Residual R = diag(lambda) w - L1 L2 (fp64) quantised per output feature n
 * in groups of G along K: INT4 s = bf16(amax / 7), q = clamp(rint(R / s),
 * -8, 7); NVFP4 s = E4M3(amax / 6 / 2^e) (satfinite), q = E2M1(R / (s 2^e)).
 * With tensor_scale (NVFP4 only) e is the smallest integer with
 * max|R| / 6 <= 448 * 2^e, else 0; *w_scale_exp (HOST int) receives e.
 * codes u8 [N x K/2] (element 2j low nibble), scales [N x K/G] (bf16 bits or
 * E4M3 bytes), written.  r may be 0 (L1, L2 unused). */
svdq_status svdq_prep_residual_quantize(svdq_variant variant, const void* w, const float* lambda,
                                        const uint16_t* L1, const uint16_t* L2, int64_t K, int64_t N,
                                        int64_t r, int tensor_scale, uint8_t* codes, void* scales,
                                        int32_t* w_scale_exp, void* stream);

/*
 * Failure reporting (no counterpart on the pages).
 * Synchronise `stream` and report device-side failures recorded by earlier
 * calls on this handle (SVDQ_ERR_DEVICE_TIMEOUT), clearing the record.
 */
svdq_status svdq_device_status(svdq_weights_t h, void* stream);

/*
 * Bit-reproducible T (no counterpart on the pages): with on = 1 the split
 * partial T tiles of kernel 1 are summed in a fixed order through a scratch
 * buffer owned by the handle (allocated here, sms * 128 * r floats plus one
 * counter per 128-row block), so T and Y are the same bits on every call
 * with the same input; with on = 0 (the default) they are added into T with
 * fp32 reductions, which is faster.  Codes and scales are bit-exact either
 * way.  Returns SVDQ_ERR_OOM if the scratch cannot be allocated, and
 * SVDQ_ERR_INVALID_ARG for on other than 0 / 1 or a different current device.
 */
svdq_status svdq_set_deterministic(svdq_weights_t h, int on);

/*
 * Failure reporting (no counterpart on the pages): the wait-site code of the
 * first bounded wait that expired in a call on this handle since the last
 * svdq_device_status (0 if none), without clearing it.  The codes identify
 * the kernel and the wait inside it; they are for diagnosis only.
 * Synchronises `stream`.
 */
svdq_status svdq_device_error_site(svdq_weights_t h, void* stream, int* site);

/*
 * Test hook (no counterpart on the pages): make the next launches wait on a
 * pipeline stage that is never filled (mask bit 0: GEMM producer skips one stage; bit 1: activation
 * kernel producer skips one stage) and use `timeout_us` as the bounded-wait
 * limit (0 restores the default of 2 s).  The kernels then return early and
 * record SVDQ_ERR_DEVICE_TIMEOUT; no GPU fault is involved.
 */
svdq_status svdq_debug_set_fault(svdq_weights_t h, uint32_t mask, uint32_t timeout_us);

/*
 * Test hook (no counterpart on the pages).
 * Self-test of the activation quantiser's division (x / s is computed with a
 * reciprocal and one fma correction step).  Runs it against IEEE fp32
 * division for every bf16 dividend and every positive finite scale of
 * `variant` (0: bf16 scales, 1: E4M3 scales) with |x / s| <= 8 on the
 * current device and writes two counts to mismatches[0..1]:
 *   [0] pairs whose 4-bit codes differ (0 expected: the codes the kernels
 *       write are exactly those of IEEE division);
 *   [1] pairs whose quotients differ while |IEEE quotient| >= 2^-24, plus
 *       the group-scale divisions amax/6 and amax/7 that differ, over all
 *       finite bf16 amax.
 * Synchronises the device.
 */
svdq_status svdq_selftest_division(int variant, unsigned long long* mismatches);

/* Human-readable name of a status code (static storage); no counterpart on
 * the pages. */
const char* svdq_status_string(svdq_status s);

/* Library version, e.g. "svdq 0.2.0 sm_100a"; no counterpart on the pages. */
const char* svdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
