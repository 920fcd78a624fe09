/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 linear layer.
 *
 * The layer computes
 *     Y = Xhat L1 L2 + Q4(Xhat) Q4(R)^T + b,   Xhat = X diag(1/lambda),
 *     R = W diag(lambda) - (L1 L2)^T,
 * where W (N x K, nn.Linear layout) is split offline into a rank-r bf16 branch
 * L1 (K x r), L2 (r x N) and a residual R quantised to NVFP4 (E2M1 codes, one
 * E4M3 scale per 16 consecutive elements along K).  Activations are quantised
 * to NVFP4 on every call; the bulk of the work runs as a 4-bit x 4-bit
 * block-scaled GEMM on the tensor cores and the low-rank correction in 16 bit.
 * A weight may instead be bound in the layer's INT4 format (signed 4-bit codes,
 * one fp16 scale per 64 elements; see svdq_weight), which every entry point
 * then follows.
 *
 * Sources of the operation (web pages on SVDQuant / Nunchaku):
 *   - W4A4, activation outliers migrated into the weights, the hard part as a
 *     16-bit low-rank branch and the rest in 4 bit: aiphreaks.com "Bringing
 *     Nunchaku 4-bit Diffusion Inference to Diffusers", section "Technical
 *     Breakdown and Performance Metrics"; chaosnode.de "Nunchaku Lite: 4-Bit
 *     Diffusion-Inferenz direkt in Diffusers", section "Die Technik: SVDQuant".
 *   - low-rank component plus residual, most work in 4-bit tensor cores and
 *     the correction in higher precision: imaginepro.ai "Nunchaku 4-Bit
 *     Diffusion Inference in Diffusers: A Practical Guide", section "Under
 *     the Hood: 4-Bit Quantization for Diffusion Models".
 *   - NVFP4 on Blackwell / B200: chaosnode.de, section "Hardware-Support";
 *     rank 32: watch-ia.com checkpoint name "...nunchaku-lite-nvfp4_r32...".
 *   - drop-in replacement of a linear layer (patched nn.Linear), offline
 *     quantisation separate from inference: chaosnode.de, section "Nunchaku
 *     Lite vs. Original"; watch-ia.com (diffuse-compressor four-step flow).
 *
 * Conventions (all entry points):
 *   - Tensors are row-major.  bf16 values are passed as uint16_t bit patterns.
 *   - "device" pointers must be CUDA device memory on the device that is
 *     current for the calling thread; they must be 16-byte aligned
 *     (SVDQ_ERR_MISALIGNED otherwise).  The caller owns every buffer.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Compute calls are asynchronous on it and never synchronise,
 *     except where stated (export, device status).
 *   - Shape limits of the GPU path: K % 256 == 0, N % 128 == 0, r % 8 == 0,
 *     0 <= r <= 64 and r <= min(N, K) (SVDQ_ERR_UNSUPPORTED_SHAPE otherwise);
 *     K % 16 != 0, N <= 0, K <= 0 or M < 0 is SVDQ_ERR_INVALID_ARG.  M == 0
 *     is a valid empty call that does nothing.  M, N, K < 2^31.
 *   - Errors are returned as status codes; nothing is thrown across the ABI.
 *     A CUDA launch/runtime failure is SVDQ_ERR_CUDA (its text is kept in a
 *     thread-local string, see svdq_last_error_detail).
 *   - The library keeps no state between calls apart from a per-device status
 *     word that kernels set when a bounded wait times out
 *     (svdq_get_device_status): bit 0 = timeout, bits 8-15 = kernel
 *     (1 activation, 2 GEMM, 3 prepare, 4 self-test, 5 INT4 kernels), bits
 *     16-23 = wait site.  Every wait gives up after 1 s.  Two entry points
 *     also own per-device resources created on first use: the copy-out stream
 *     and events of svdq_linear_forward_host (concurrent callers on one device
 *     enqueue one after the other) and the scratch of
 *     svdq_linear_forward_noalloc.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, negative or non-multiple-of-16 size */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* valid layer, but outside the GPU path's limits   */
  SVDQ_ERR_MISALIGNED = 3,         /* a device pointer is not 16-byte aligned           */
  SVDQ_ERR_WORKSPACE_TOO_SMALL = 4,
  SVDQ_ERR_CUDA = 5,               /* CUDA runtime / launch error                       */
  SVDQ_ERR_TIMEOUT = 6,            /* a kernel's bounded wait expired (device status)   */
  SVDQ_ERR_SOLVER = 7              /* the eigen-solver of svdq_prepare_weight failed    */
} svdq_status;

/*
 * A prepared layer.  All pointers are device pointers owned by the caller
 * (svdq_weight_bind carves them out of one buffer).  Layouts:
 *   w_codes    N x K/2 bytes: NVFP4 codes of R, row n holds R[n, :], element
 *              2j in the low nibble of byte j (E2M1: bit 3 sign, bits 0-2
 *              magnitude index into {0,.5,1,1.5,2,3,4,6}).
 *   w_scales   E4M3 scale codes of R in the scale-factor tile layout used by
 *              the block-scaled tensor-core MMA: 512-byte tiles of 128 rows x
 *              4 scales (64 K-elements); tile (rb, kb) at byte
 *              (rb * K/64 + kb) * 512, and inside a tile, row i and scale j at
 *              (i % 32) * 16 + (i / 32) * 4 + j.  Size N * K / 16 bytes.
 *   L1         K x r bf16, L1 = U_r diag(sigma_r) of the smoothed weight.
 *   L1f        the same K x r values in the B-fragment order of the warp-level
 *              bf16 MMA m16n8k16 (read by the activation kernel): for k-step
 *              g = k/16 and column tile t = j/8, the 32 lanes' fragments follow
 *              each other; 32-bit word ((g * r/8 + t) * 32 + lane) * 2 + h holds
 *              L1[16g + 2(lane%4) + 8h + {0 (low half), 1}][8t + lane/4].
 *   L2t        N x r bf16, L2^T = V_r.
 *   inv_lambda K float32, f32(1 / lambda).
 *   bias       N bf16, or NULL when has_bias == 0.
 *   L1t        r x K bf16, L1 transposed (row j holds L1[:, j]; read by the
 *              layer's activation kernel, whose tensor-core product with the
 *              activation tile needs L1 with K contiguous).  Written, like
 *              L1f, by svdq_prepare_weight and svdq_weight_import.
 *
 * INT4 format (format == SVDQ_FORMAT_INT4): the other 4-bit format of the
 * layer, used before Blackwell (chaosnode.de "Nunchaku Lite", section
 * "Hardware-Support").  w_codes has the same N x K/2 shape and nibble order,
 * the nibbles being two's-complement integers in [-8, 7]; w_scales holds one
 * fp16 scale per group of 64 elements along K, group-major: fp16 [K/64][N]
 * (scale of row n, group g at element g * N + n; N * K / 32 bytes, a prefix
 * of the field).  Quantiser of a group v[64]: s = fp16_RNE(min(f32(max|v| /
 * 7), 65504)), q = clamp(RNE(f32(v / s)), -8, 7), q = 0 when s == 0.  All
 * other fields are shared with NVFP4.
 */
#define SVDQ_FORMAT_NVFP4 0
#define SVDQ_FORMAT_INT4 1

typedef struct svdq_weight {
  int32_t N, K, r;
  int32_t has_bias;
  int32_t format;     /* SVDQ_FORMAT_NVFP4 (default of svdq_weight_bind) or SVDQ_FORMAT_INT4 */
  uint8_t* w_codes;
  uint8_t* w_scales;
  uint16_t* L1;
  uint16_t* L1f;
  uint16_t* L2t;
  float* inv_lambda;
  uint16_t* bias;
  uint16_t* L1t;
} svdq_weight;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(svdq_status s);

/* Text of the last SVDQ_ERR_CUDA / SVDQ_ERR_SOLVER seen on this host thread. */
const char* svdq_last_error_detail(void);

/* Library version, e.g. "svdq-b200 0.1". */
const char* svdq_version(void);

/* ---------------------------------------------------------------------------
 * Sizes.  Pure host functions; 0 means the shape is invalid or unsupported.
 * ------------------------------------------------------------------------- */

/* Bytes of one svdq_weight buffer (all fields, each 256-byte aligned). */
size_t svdq_weight_bytes(int N, int K, int r, int has_bias);

/* Bytes of activation codes (M x K/2), scales (M rounded up to 128 rows, in
 * the scale-factor tile layout above) and D (M x r bf16). */
size_t svdq_act_codes_bytes(int M, int K);
size_t svdq_act_scales_bytes(int M, int K);

/* Workspace of svdq_linear_forward (and its host, head-major and no-allocation
 * variants), 256-byte aligned fields.  For the general path: codes (M x K/2),
 * scales (tile layout above) and D (M x r bf16), then, for r > 0, the
 * activation kernel's K-split partials of D (float32, 8 roundup(M,128) r)
 * and their flags (uint64 [roundup(M,128)/128][8]; see svdq_quantize_act_ws;
 * their contents need not be initialised).  For M <= 32 and K <= 3840
 * the few-token path (see svdq_linear_forward) uses, from the start of the
 * same buffer: codes M x K/2; the scale words uint32 [K/64][32] (word j of
 * token m holds the E4M3 codes of its 16-element blocks 4 j .. 4 j + 3, low
 * byte first; tokens >= M are 0); the float32 partial down-projections
 * [K/256][M][r] (D = bf16 of their sum in slice order).  The size returned
 * covers both. */
size_t svdq_forward_workspace_bytes(int M, int N, int K, int r);

/* Workspace of svdq_prepare_weight.  This asks the eigen-solver for its
 * buffer size and therefore needs a CUDA device (returns 0 without one). */
size_t svdq_prepare_workspace_bytes(int N, int K, int r);

/* Carve a caller-allocated device buffer of svdq_weight_bytes() bytes into the
 * fields of *out (pointer arithmetic only, no device access). */
svdq_status svdq_weight_bind(void* buf, size_t bytes, int N, int K, int r, int has_bias,
                             svdq_weight* out);

/* svdq_weight_bind, then out->format = format (SVDQ_FORMAT_NVFP4 or
 * SVDQ_FORMAT_INT4; anything else is SVDQ_ERR_INVALID_ARG).  Every entry point
 * that takes the weight follows its format. */
svdq_status svdq_weight_bind_format(void* buf, size_t bytes, int N, int K, int r, int has_bias, int format,
                                    svdq_weight* out);

/* ---------------------------------------------------------------------------
 * Offline preparation (smoothing, rank-r split, residual NVFP4 pack).
 * Defined by: outliers migrated from the activations into the weights, then
 * absorbed by a 16-bit low-rank branch with the rest quantised to 4 bit
 * (chaosnode.de "Nunchaku Lite", section "Die Technik: SVDQuant";
 * aiphreaks.com, section "Technical Breakdown and Performance Metrics"); the
 * weight split into a low-rank component and a residual (imaginepro.ai,
 * section "Under the Hood"); quantisation as a separate offline step
 * (watch-ia.com, the diffuse-compressor flow).
 *   W       device, N x K bf16 (nn.Linear weight)
 *   lambda  device, K float32 smoothing factors (> 0, finite), calibrated by
 *           the caller from activation statistics
 *   bias    device, N bf16, or NULL (must be non-NULL iff w->has_bias)
 *   w       weight bound with svdq_weight_bind for the same N, K, r
 *   ws      device workspace of svdq_prepare_workspace_bytes() bytes
 * Steps: What = f32(W * lambda) per column; L1 = U_r diag(sigma_r),
 * L2 = V_r^T from the top-r eigenpairs of the float64 Gram matrix of What
 * (the smaller of What What^T and What^T What), each pair sign-normalised so
 * the largest-|.| entry of u_i is positive, stored as bf16 (RNE);
 * R = f32(What - (bf16 L1 bf16 L2)^T) summed in float64; R quantised to NVFP4
 * along K (to INT4 groups of 64 when w->format == SVDQ_FORMAT_INT4).  Offline: it creates (and destroys) one cuSOLVER handle per call,
 * whose own small allocation is the one exception to "never allocates", and
 * the solver may synchronise the stream.
 * ------------------------------------------------------------------------- */
svdq_status svdq_prepare_weight(const uint16_t* W, const float* lambda, const uint16_t* bias,
                                const svdq_weight* w, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Activation kernel (one HBM pass over X).
 * Defined by: the activations quantised to 4 bit on every call once the
 * outliers have moved into the weights ("A4" of W4A4: aiphreaks.com, section
 * "Technical Breakdown and Performance Metrics"; watch-ia.com, W4A4), and the
 * 16-bit low-rank branch's input projection (imaginepro.ai, "Under the Hood").
 *   X        device, M x K bf16
 *   x_codes  device, M x K/2 NVFP4 codes of Xhat = f32(X * inv_lambda)
 *   x_scales device, svdq_act_scales_bytes(M, K) bytes, tile layout; rows
 *            M .. roundup(M,128)-1 are written as zero
 *   D        device, M x r bf16, D = bf16(sum_k bf16(Xhat)_mk bf16(L1)_kj)
 *            with float32 accumulation; may be NULL when r == 0
 * With an INT4 weight the codes are INT4 and x_scales holds fp16 group scales
 * group-major, [K/64][roundup(M,128)] (scale of row m, group g at element
 * g * roundup(M,128) + m; padding rows zero); the buffer size above covers it.
 * ------------------------------------------------------------------------- */
svdq_status svdq_quantize_act(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                              uint8_t* x_scales, uint16_t* D, void* stream);

/* The same outputs through the activation kernel that svdq_linear_forward
 * runs: for r > 0 and enough work per CTA (each of the 128-row CTAs, K split
 * across up to 8 of them, walks at least 12 stages of 64 columns) a kernel
 * with D on the tensor cores, which needs a workspace for the K split's
 * float32 partials of D and their flags; otherwise svdq_quantize_act's.
 *   ws        device, at least svdq_act_workspace_bytes(M, K, r) bytes
 *             (256 bytes when r == 0), contents need not be initialised
 * Codes and scales equal those of svdq_quantize_act bit for bit; D may
 * differ from its D by float32 summation order (both are within D's bound),
 * and equals the D that svdq_linear_forward computes for the same X.  With
 * r == 0 or an INT4 weight this is svdq_quantize_act.  Returns 0 bytes for
 * an invalid shape. */
size_t svdq_act_workspace_bytes(int M, int K, int r);
svdq_status svdq_quantize_act_ws(const uint16_t* X, int M, const svdq_weight* w, uint8_t* x_codes,
                                 uint8_t* x_scales, uint16_t* D, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Block-scaled FP4 GEMM with the low-rank branch and bias fused:
 *   Y = bf16(deq(x_codes, x_scales) deq(w_codes, w_scales)^T + D L2 + bias),
 * float32 accumulation in tensor memory.  Inputs as produced by
 * svdq_quantize_act; Y device, M x N bf16.  Single CTAs compute 128 x 256
 * output tiles (N % 256 == 0 and at least one tile per SM) or 128 x 128 tiles
 * (SVDQ_OVERRIDE_GEMM_BN replaces that choice).
 * Defined by: "most operations happen in 4-bit tensor cores, while the
 * low-rank correction runs in higher precision" (imaginepro.ai practical
 * guide, section "Under the Hood: 4-Bit Quantization for Diffusion Models");
 * the 4-bit operands are NVFP4 on B200 (chaosnode.de, "Hardware-Support").
 * With an INT4 weight: Y = bf16(sum_g sx[m,g] sw[n,g] (sum_{k in group g}
 * qx[m,k] qw[n,k]) + D L2 + bias), the integer group sums exact (8-bit integer
 * warp MMA on the sign-extended codes) and the scaling in float32; 128 x 128
 * tiles, one CTA each.
 * ------------------------------------------------------------------------- */
svdq_status svdq_gemm(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                      const svdq_weight* w, uint16_t* Y, void* stream);

/* ---------------------------------------------------------------------------
 * The same GEMM (and whole layer, below) writing Y head-major for attention
 * consumers: Y[h][m][d] = Yrow[m][h * head_dim + d], i.e. N / head_dim blocks
 * of M x head_dim bf16, one per head (for a QKV projection: the Q heads, then
 * K, then V).  The engine the chaosnode.de page ("Nunchaku Lite vs. Original")
 * describes fuses the QKV projection with its consumers; this is the layout
 * half of that.  head_dim % 16 == 0 and N % head_dim == 0 (INVALID_ARG
 * otherwise).  The values are bit for bit those of svdq_gemm; the single-CTA
 * kernel is always used.
 * ------------------------------------------------------------------------- */
svdq_status svdq_gemm_heads(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* D, int M,
                            const svdq_weight* w, int head_dim, uint16_t* Y, void* stream);

/* Whole layer with head-major Y (see svdq_gemm_heads); workspace as for
 * svdq_linear_forward. */
svdq_status svdq_linear_forward_heads(const uint16_t* X, int M, const svdq_weight* w, int head_dim,
                                      uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Whole layer.  Defined by: the SVDQ layer as a drop-in replacement of a
 * linear layer, run W4A4 at inference (chaosnode.de "Nunchaku Lite",
 * sections "Die Technik: SVDQuant" and "Nunchaku Lite vs. Original";
 * aiphreaks.com, section "Technical Breakdown and Performance Metrics").
 * Few-token path: with an NVFP4 weight, M <= 32, K <= 3840 and N / 128 at
 * most the number of SMs, the layer is a weight stream and runs as an
 * activation kernel (K / 256 CTAs: codes, scales, partial D) and a GEMM with
 * the operands swapped (the weight's 128 rows are the MMA's M, the tokens its
 * N = 16 or 32; one CTA per 128 weight rows, weight streaming from its first
 * instruction); same results up to float32 summation order of D.
 * SVDQ_OVERRIDE_SMALL_M = 1 turns it off.  Otherwise (general path)
 * svdq_quantize_act then svdq_gemm on `stream`, with the
 * activation codes, scales and D placed in the caller's workspace `ws`
 * (svdq_forward_workspace_bytes(M, N, K, r) bytes, device).
 * ------------------------------------------------------------------------- */
svdq_status svdq_linear_forward(const uint16_t* X, int M, const svdq_weight* w, uint16_t* Y,
                                void* ws, size_t ws_bytes, void* stream);

/* Same as svdq_linear_forward but with X and Y in pinned HOST memory: copies
 * X_host -> X_dev (M x K bf16), runs the layer into Y_dev, copies Y_dev ->
 * Y_host (M x N bf16), asynchronously with respect to the host and ordered on
 * `stream` (the caller synchronises `stream` before reading Y_host).  Above
 * 1024 rows the work is split into chunks of 1024 rows: each chunk's copy
 * back to the host runs on a second, library-owned stream (one per device,
 * created on first use) while the next chunk is copied in and computed, and
 * `stream` then waits for the last copy.  ws is sized for M as for
 * svdq_linear_forward.  SVDQ_OVERRIDE_HOST_CHUNK_ROWS (a multiple of 128)
 * replaces the chunk size. */
svdq_status svdq_linear_forward_host(const uint16_t* X_host, int M, const svdq_weight* w,
                                     uint16_t* Y_host, uint16_t* X_dev, uint16_t* Y_dev,
                                     void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * MLP pair: up-projection, GELU, down-projection, both SVDQ layers, with the
 * GELU and the down-projection's activation quantisation fused into the
 * up-projection's epilogue.  Defined by: the original engine's model-specific
 * fused GELU / MLP kernels (chaosnode.de "Nunchaku Lite", section "Nunchaku
 * Lite vs. Original"); each linear as in svdq_linear_forward.
 *   H    = bf16(gelu_tanh(Y_up)),  Y_up = the up-projection's bf16 output,
 *          gelu_tanh(y) = y/2 (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))),
 *          evaluated in float32 as y / (1 + exp(-2u)) (the same function);
 *   Y    = the down-projection of H (its own smoothing, NVFP4 codes and D).
 * The up-projection's GEMM writes, per 16 hidden columns of a row, the
 * down-projection's NVFP4 codes and scale of Hhat = f32(H / lambda_down)
 * straight into that layer's activation buffers, and accumulates its
 * D = bf16(sum_k bf16(Hhat) L1_down) in float32 (tensor-core partials per
 * tile, added across tiles); H itself never crosses HBM.
 *   X      device, M x K bf16 (K = up->K)
 *   up     NVFP4 weight, N = F (the hidden width);  down: NVFP4, K = F, r <= 32
 *          (SVDQ_ERR_UNSUPPORTED_SHAPE otherwise; INVALID_ARG if K != F)
 *   Y      device, M x down->N bf16
 *   H_out  optional device M x F bf16: H is also written there (NULL: not)
 *   ws     device, svdq_mlp_workspace_bytes(M, K, F, down->N, up->r, down->r)
 *          bytes: the up-projection's activation workspace (the general
 *          layout of svdq_forward_workspace_bytes(M, F, K, up->r) bytes), the
 *          down-projection's (codes M x F/2, scales, D; the general layout of
 *          svdq_forward_workspace_bytes(M, N, F, down->r) bytes, both rounded
 *          up to 256), then M x down->r float32.
 * Asynchronous on `stream`; the two GEMMs' results equal the unfused pair's
 * up to the float32 evaluation of GELU (one bf16 step of H next to a rounding
 * boundary) and the summation order of D.
 * ------------------------------------------------------------------------- */
size_t svdq_mlp_workspace_bytes(int M, int K, int F, int N, int r_up, int r_down);
svdq_status svdq_mlp_forward(const uint16_t* X, int M, const svdq_weight* up, const svdq_weight* down, uint16_t* Y,
                             uint16_t* H_out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Whole layer for callers that cannot allocate device memory.  The pages have
 * no counterpart of this entry point: it is an interface convenience.
 *
 * Some callers cannot call cudaMalloc or receive a workspace: plugin or
 * extension hosts that hand a layer only its input and output buffers and keep
 * the device allocator to themselves (an allocation there would bypass the
 * host's memory pool and its accounting), and latency-critical loops in which
 * cudaMalloc / cudaFree would synchronise the device.  For them this variant
 * of svdq_linear_forward takes the activation codes, scales and D from a
 * fixed scratch array that the library holds in device memory (a file-scope
 * __device__ array of SVDQ_NOALLOC_SCRATCH_BYTES bytes, resident on every GPU
 * that loads the library until the process exits).  It calls no allocator.
 *   X, Y    device, as for svdq_linear_forward (caller-owned).
 *   Shapes whose workspace (svdq_forward_workspace_bytes) exceeds the scratch
 *   are rejected with SVDQ_ERR_WORKSPACE_TOO_SMALL and a message in
 *   svdq_last_error_detail.
 *   The first call on a device looks up the scratch's device address (with
 *   that device current) and caches it; make that first call before any
 *   stream capture.
 *   Every call shares the one scratch array, which keeps the last call's
 *   contents: calls whose kernels overlap on the GPU (different streams, or
 *   several threads) race on it.  Each call overwrites every scratch byte it
 *   later reads, so nothing needs clearing between calls.
 * ------------------------------------------------------------------------- */
#define SVDQ_NOALLOC_SCRATCH_BYTES (64u << 20)
svdq_status svdq_linear_forward_noalloc(const uint16_t* X, int M, const svdq_weight* w,
                                        uint16_t* Y, void* stream);

/* ---------------------------------------------------------------------------
 * Defined by: the offline flow's "package" step, a quantised checkpoint that
 * is later loaded and verified (watch-ia.com, the diffuse-compressor flow).
 * Test / checkpoint path: copy a prepared weight to host buffers in logical
 * layouts (codes N x K/2, scales N x K/16 row-major, L1 K x r, L2t N x r,
 * inv_lambda K).  For an INT4 weight the scales are N x K/64 fp16 (uint16
 * bit patterns, N * K / 32 bytes), row-major.  Any host pointer may be NULL to
 * skip that field.  Synchronises `stream`.
 * ------------------------------------------------------------------------- */
svdq_status svdq_weight_export(const svdq_weight* w, uint8_t* host_codes, uint8_t* host_scales,
                               uint16_t* host_L1, uint16_t* host_L2t, float* host_inv_lambda,
                               void* stream);

/* Checkpoint import, the inverse of svdq_weight_export: fill a bound weight
 * from host buffers in the same logical layouts (codes N x K/2, scales
 * N x K/16 row-major -- N x K/64 fp16 for an INT4 weight -- L1 K x r, L2t N x r,
 * inv_lambda K) plus the bias (N bf16; required exactly when w->has_bias).  The
 * scales are converted to the native layout on the host and L1f is regenerated
 * from L1 on the device.  The
 * watch-ia.com page's offline loop ("quantise, package, load and verify")
 * needs this load step.  Synchronises `stream`.  SVDQ_ERR_INVALID_ARG for a
 * missing buffer. */
svdq_status svdq_weight_import(const svdq_weight* w, const uint8_t* host_codes, const uint8_t* host_scales,
                               const uint16_t* host_L1, const uint16_t* host_L2t,
                               const float* host_inv_lambda, const uint16_t* host_bias, void* stream);

/* Calibration statistics (offline): colmax[k] = max(colmax[k], max_m |A[m][k]|)
 * for a device rows x K bf16 matrix A, row-major.  colmax is a device float
 * array of K entries; zero it before the first batch, then call once per
 * calibration batch of activations.  Asynchronous on `stream`. */
svdq_status svdq_calib_absmax(const uint16_t* A, int rows, int K, float* colmax, void* stream);

/* Smoothing factors from calibration statistics (offline):
 *   lambda[k] = f32( x_k^alpha / w_k^(1 - alpha) ),  x_k = x_absmax[k],
 *   w_k = max_n |W[n][k]|, evaluated in float64; alpha = 0.5 is evaluated as
 *   f32(sqrt(x_k / w_k)); lambda[k] = 1 where x_k or w_k is 0.
 * alpha in [0, 1] is the migration strength: the share of each input
 * channel's activation range moved into the weight (0.5 balances the two
 * maxima).  W device N x K bf16; x_absmax and lambda device, K floats.
 * Asynchronous on `stream`; lambda is then the input of svdq_prepare_weight. */
svdq_status svdq_calibrate_lambda(const float* x_absmax, const uint16_t* W, int N, int K, float alpha,
                                  float* lambda, void* stream);

/* Host-only layout conversions between logical [rows][K/16] scales and the
 * tile layout (rows of the tile layout are `rows` rounded up to 128; padding
 * entries are written as 0 by to_native and ignored by to_logical). */
svdq_status svdq_scales_to_logical(const uint8_t* native, int rows, int K, uint8_t* logical);
svdq_status svdq_scales_to_native(const uint8_t* logical, int rows, int K, uint8_t* native);

/* The activation scales of svdq_quantize_act (M token rows) in logical
 * [M][K/16] order: svdq_scales_to_logical under the name the interface's
 * checkpoint/test tooling uses. */
svdq_status svdq_act_scales_to_logical(const uint8_t* native, int M, int K, uint8_t* logical);

/* Host-only conversions of INT4 fp16 scales between the logical [rows][K/64]
 * layout and the group-major [K/64][rows_pad] one (rows_pad >= rows: N for a
 * weight, roundup(M,128) for activations; padding written as 0). */
svdq_status svdq_int4_scales_to_logical(const uint16_t* native, int rows, int rows_pad, int K,
                                        uint16_t* logical);
svdq_status svdq_int4_scales_to_native(const uint16_t* logical, int rows, int rows_pad, int K,
                                       uint16_t* native);

/* ---------------------------------------------------------------------------
 * Overrides of automatic launch choices, for tests and tuning sweeps.  The
 * pages have no counterpart: this is test support.  Process-wide (every
 * device, every thread); value 0 restores the automatic choice.  Nothing else
 * (no environment variable) changes these choices.
 *   SVDQ_OVERRIDE_ACT_KSPLIT       CTAs sharing a 16-row block of the
 *                                  activation kernel (1-8; used when K is a
 *                                  multiple of 64 x value)
 *   SVDQ_OVERRIDE_GEMM_BN          GEMM tile width 128 or 256 (256 only when
 *                                  N % 256 == 0)
 *   SVDQ_OVERRIDE_HOST_CHUNK_ROWS  rows per chunk of svdq_linear_forward_host
 *                                  (a multiple of 128)
 *   SVDQ_OVERRIDE_SMALL_M          1 = never take the few-token path of
 *                                  svdq_linear_forward (see there)
 *   SVDQ_OVERRIDE_ACT_KERNEL       activation kernel of svdq_linear_forward
 *                                  and svdq_quantize_act_ws for r > 0: 1 = the
 *                                  16-row kernel, 2 = the 128-row kernel with
 *                                  D on the tensor cores
 * Results are identical under every setting up to float32 summation order
 * (the tests check each against the oracle).  SVDQ_ERR_INVALID_ARG for an
 * unknown `which` or a negative value.
 * ------------------------------------------------------------------------- */
#define SVDQ_OVERRIDE_ACT_KSPLIT 1
#define SVDQ_OVERRIDE_GEMM_BN 2
#define SVDQ_OVERRIDE_HOST_CHUNK_ROWS 3
#define SVDQ_OVERRIDE_SMALL_M 4
#define SVDQ_OVERRIDE_ACT_KERNEL 5
#define SVDQ_OVERRIDE_COUNT 6
svdq_status svdq_set_override(int which, int value);

/* Synchronise `stream` and report the device status word of the current
 * device: SVDQ_OK, or SVDQ_ERR_TIMEOUT if a kernel gave up a bounded wait
 * since the last clear.  *detail (optional) receives the raw word. */
svdq_status svdq_get_device_status(void* stream, uint32_t* detail);
svdq_status svdq_clear_device_status(void* stream);

/* Failure-detection self-test: launch one bounded wait (the same kind every
 * kernel of the library uses) on an mbarrier that nothing completes, with the
 * given limit in nanoseconds (clamped to [1 us, 1 s]).  The wait gives up,
 * records a timeout (kernel id 4, site 1) in the device status word and the
 * kernel returns normally: the context stays usable.  Asynchronous on
 * `stream`; read the result with svdq_get_device_status. */
svdq_status svdq_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Numerics self-test of the activation kernel's quantiser on the current
 * device (synchronous, default stream).  The kernel takes each element's code
 * from RN(v / s) computed without a division (one multiply by RN(1/s) and the
 * FMA quotient correction of Markstein, IBM J. Res. Dev. 34(1), 1990).  This
 * runs that exact device routine for every E4M3 scale s > 0, both signs, five
 * binades of v around s and all 2^23 significands of v, plus signed zeros,
 * subnormal, tiny, huge and tie values for every scale code including s = 0
 * (whose quotient is defined as a zero with v's sign), and writes
 * counts[0] = quotients differing from IEEE float32 division where that
 * quotient is normal or zero, counts[1] = E2M1 codes (sign bit kept)
 * differing from the format's definition applied to the IEEE quotient, and
 * counts[2] = quotient differences where the IEEE quotient is subnormal (the
 * correction step is not exact there, but such quotients lie far below the
 * first E2M1 threshold 0.25, so their codes are checked by counts[1]).
 * counts[0] and counts[1] are 0 on a correct build.  `counts` is a host array
 * of 3.  The paper has no counterpart: this is test support. */
svdq_status svdq_selftest_quotient(uint64_t* counts);

/* Numerics self-test of the hardware conversions the kernels round with, on
 * the current device (synchronous).  For every non-negative finite float32 x
 * it compares cvt.rn.satfinite.e4m3x2 with the nearest of the 127 finite E4M3
 * values (ties to the even code, saturating at 448), cvt.rn.satfinite.e2m1x2
 * with the E2M1 thresholds 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5 (ties to even),
 * and cvt.rn.bf16x2 with round-to-nearest-even on the upper 16 bits, and
 * writes the mismatch counts to counts[0..2] (host array of 3; all 0 on a
 * correct device).  The paper has no counterpart: this is test support. */
svdq_status svdq_selftest_conversions(uint64_t* counts);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* SVDQ_H_ */
