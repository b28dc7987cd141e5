/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 W4A4 linear-layer kernels for
 * NVIDIA B200 (sm_100a).
 *
 * Two core operations, both asynchronous on a caller-supplied CUDA stream
 * (variants declared further down: a static tensor scale, quantization of
 * x^T, ARCQuant augmented residual channels, an allocation-free quantizer,
 * per-segment B scales, a GEMM that writes an NVFP4 output, and one call that
 * quantizes the activations and runs the GEMM):
 *
 *  nvfp4_quantize  16-element block-scaled NVFP4 quantization of a bf16
 *                  matrix: E2M1 codes, one FP8 E4M3 scale per 16 elements
 *                  along K, one FP32 global scale per tensor.  Two modes:
 *                  scale-to-6 and the adaptive Four-Over-Six (4/6), which
 *                  quantizes every block with scale targets 6 and 4 and keeps
 *                  the one with the smaller error under a max / MAE / MSE rule.
 *                  Source: "Four Over Six (4/6)" technical summary,
 *                  gist.science/ko/paper/2512.02010 -- sections "문제 제기"
 *                  (E2M1 grid 0,.5,1,1.5,2,3,4,6), "적응형 블록 스케일링
 *                  알고리즘" (double quantization, three selection rules) and
 *                  "구현 세부 사항" (E4M3 block scales; FP8 max 256 instead of
 *                  448 in the global scale for 4/6).
 *
 *  nvfp4_gemm      Y = alpha_A * alpha_B * sum_kb sA[m,kb] sB[n,kb] *
 *                      sum_{k in kb} qA[m,k] qB[n,k]
 *                  i.e. Y = A_hat . B_hat^T for two NVFP4 operands stored as
 *                  nvfp4_quantize writes them, both K-major, with an fp32
 *                  accumulator and a bf16 or fp32 output.  Source: "ARCQuant"
 *                  technical summary, gist.science/ko/paper/2601.07475,
 *                  section "방법론" (one uniform NVFP4 GEMM along K on the
 *                  Blackwell tensor cores), and the Minima page, section
 *                  "심층 분석" (global scales applied around one fused GEMM).
 *
 * Exact arithmetic of nvfp4_quantize (every step one IEEE binary32 operation,
 * round-to-nearest-even, in this order):
 *   amax  = max |x| over the tensor
 *   alpha = amax / (fp8_max * 6)            (alpha = 1 when amax == 0)
 *   per block of 16 along K, b = max |x_i|, for Q in {6} or {6, 4}:
 *     s = E4M3_RNE_satfinite(b / (alpha * Q));  d = s * alpha
 *     r = 1 / d, or 0 when that is infinite;    v_i = x_i * r
 *     q_i = E2M1_RNE_satfinite(v_i) (sign kept); e_i = fma(-q_i, d, x_i)
 *     E_Q = max|e_i| (MAX), sum |e_i| (MAE) or sum e_i*e_i (MSE), sums as
 *           the contiguous pairwise tree ((e0+e1)+(e2+e3))+...
 *   keep Q = 4 only when E_4 < E_6.
 *
 * Memory layouts (all buffers are device memory owned by the caller; the
 * library allocates nothing and keeps no pointer after a call returns):
 *   x       bf16 [rows, K], row stride ldx elements (ldx >= K, ldx % 8 == 0,
 *           base 16-byte aligned).
 *   codes   uint8 [rows, K/2], row-major, two E2M1 codes per byte, element 2j
 *           in the low nibble (nvfp4_codes_bytes).  16-byte aligned.
 *   scales  E4M3 bytes in the block-scaled MMA's scale-factor layout: atoms
 *           of 128 rows x 4 K-blocks (64 elements), 512 bytes each, atom
 *           (r/128)*(K/64) + (k/64), byte (r%32)*16 + ((r/32)%4)*4 + (k/16)%4
 *           inside the atom; rows padded to a multiple of 128 with zero bytes
 *           (nvfp4_scales_bytes).  16-byte aligned.
 *   global_scale  one fp32 in device memory (alpha).
 *   Y       bf16 or fp32 [M, N], row-major, row stride ldy >= N elements,
 *           aligned to its element size.  When its base and row pitch are
 *           16-byte aligned the epilogue stores through TMA, otherwise with
 *           direct stores.
 *
 * Errors: every call validates its arguments on the host and returns a status
 * without launching anything when they are invalid.  Conditions only the GPU
 * can see (non-finite input to nvfp4_quantize, a static alpha that is not a
 * positive finite number, a bounded device wait that ran out) are
 * written to a status word in the call's workspace and read by
 * nvfp4_get_device_status.  Launch failures return NVFP4_ERR_CUDA with
 * the CUDA message available from nvfp4_last_error_message.
 *
 * Streams are passed as void* and must be a cudaStream_t of the current
 * device (NULL = the legacy default stream).  All calls use the current CUDA
 * device of the calling thread.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,        /* null pointer, bad size, alignment, enum value */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 2, /* current device is not compute capability 10.0 */
  NVFP4_ERR_NONFINITE = 3,          /* input tensor holds Inf or NaN (device status) */
  NVFP4_ERR_TIMEOUT = 4,            /* a bounded device wait ran out (device status) */
  NVFP4_ERR_CUDA = 5                /* a CUDA runtime / driver call failed */
} nvfp4_status;

typedef enum { NVFP4_MODE_SIX = 0, NVFP4_MODE_FOUR_OVER_SIX = 1 } nvfp4_mode;
typedef enum { NVFP4_RULE_MAX = 0, NVFP4_RULE_MAE = 1, NVFP4_RULE_MSE = 2 } nvfp4_rule;
typedef enum { NVFP4_OUT_BF16 = 0, NVFP4_OUT_FP32 = 1 } nvfp4_out_dtype;

/* Bytes of the packed code buffer: rows * K / 2. */
NVFP4_API size_t nvfp4_codes_bytes(int64_t rows, int64_t K);

/* Bytes of the swizzled scale buffer: ceil(rows/128)*128 * K/16. */
NVFP4_API size_t nvfp4_scales_bytes(int64_t rows, int64_t K);

/* Bytes of device workspace nvfp4_quantize needs (a status word and the
 * per-CTA partial maxima of the tensor-amax pass).  Any size-independent
 * workspace of at least this many bytes, 16-byte aligned, may be reused
 * across calls on one stream; calls that run concurrently need their own. */
NVFP4_API size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K);

/* Bytes of device workspace nvfp4_gemm needs (its status word). */
NVFP4_API size_t nvfp4_gemm_workspace_bytes(void);

/* Quantize x [rows, K] (bf16) to NVFP4.
 *   mode     NVFP4_MODE_SIX or NVFP4_MODE_FOUR_OVER_SIX.
 *   rule     selection rule for 4/6 (NVFP4_RULE_*); ignored for SIX but must
 *            still be a valid value.
 *   fp8_max  448 or 256: the FP8 maximum used in alpha = amax/(fp8_max*6).
 *            The pages use 448 for scale-6 and 256 for 4/6; any pairing is
 *            accepted.
 * Requirements: rows >= 1, K >= 64, K % 64 == 0, ldx >= K, ldx % 8 == 0,
 * rows * ldx <= 2^40 and (rows rounded up to 128) * (K rounded up to 512)
 * < 2^40 elements,
 * x / codes / scales / workspace 16-byte aligned, global_scale 4-byte
 * aligned, workspace_bytes >= nvfp4_quantize_workspace_bytes(rows, K).
 * Writes codes, every byte of scales (padding = 0), *global_scale and the
 * workspace status word.  When x holds Inf or NaN the status word becomes
 * NVFP4_ERR_NONFINITE, *global_scale becomes NaN, and codes/scales are left
 * unwritten.  Returns once both kernels are enqueued: the amax pass, then the
 * quantize kernel as its programmatic dependent (scheduled while the amax pass
 * drains; it waits for the pass before reading anything). */
NVFP4_API nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                            int rule, float fp8_max, void* codes, void* scales,
                            float* global_scale, void* workspace, size_t workspace_bytes,
                            void* stream);

/* Augmented residual channels (ARCQuant page, "기술 요약" / "방법론"): the
 * NVFP4 operand of the [rows, K + S] matrix whose first K channels are the
 * channels of x in the order perm (outlier channels first, as calibration
 * ranks them) and whose last S channels are
 *   augment = 0: the residual e = x - q*d of the first S reordered channels
 *                against their own quantization (activations), or
 *   augment = 1: a copy of the first S reordered channels (the weight, whose
 *                matching columns are duplicated),
 * all quantized with the same alpha (the amax of x), mode and rule, so that
 * one nvfp4_gemm over K + S adds the residual correction in its accumulator.
 *   perm    device int32[K], a permutation of 0..K-1 (entries outside 0..K-1
 *           are read as channel 0)
 *   S       0 <= S <= K, S % 64 == 0
 *   codes   [rows, (K+S)/2];  scales  nvfp4_scales_bytes(rows, K + S)
 * Requirements otherwise as nvfp4_quantize, and K <= 16384 (rows and the
 * permutation are staged in shared memory).  Two kernel launches. */
NVFP4_API nvfp4_status nvfp4_quantize_arc(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                          const int32_t* perm, int64_t S, int augment, int mode, int rule,
                                          float fp8_max, void* codes, void* scales, float* global_scale,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* nvfp4_quantize_arc with the RMSNorm of the activations fused ahead of it
 * (ARCQuant page, "방법론", 커널 구현: the fused kernel normalizes, reorders
 * and quantizes the primary and residual channels): the operand is that of
 * nvfp4_quantize_arc (augment = 0) applied to the bf16 tensor
 *   y[i, k] = bf16((x[i, k] * r_i) * gamma[k]),
 *   r_i = 1 / sqrt(sum_k x[i, k]^2 / K + eps),
 * every step one binary32 operation, the sum of squares taken as the
 * contiguous pairwise tree over the row (zero-padded to a power of two), the
 * square root and the divisions correctly rounded.  alpha is the amax of y.
 * y is never written: a row pass computes r_i and the amax partials, and
 * copies gamma into channel order (both kept in the workspace), and the
 * augmented quantizer normalizes the channels it gathers.
 *   gamma   device bf16[K], 16-byte aligned
 *   eps     a positive finite number
 *   workspace  nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K) bytes
 * Other arguments and requirements as nvfp4_quantize_arc.  A non-finite y
 * (from non-finite x, or a product past the bf16 range) sets
 * NVFP4_ERR_NONFINITE as for nvfp4_quantize.  Two kernel launches. */
NVFP4_API size_t nvfp4_quantize_arc_rmsnorm_workspace_bytes(int64_t rows, int64_t K);
NVFP4_API nvfp4_status nvfp4_quantize_arc_rmsnorm(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                                  const void* gamma, float eps, const int32_t* perm, int64_t S,
                                                  int mode, int rule, float fp8_max, void* codes, void* scales,
                                                  float* global_scale, void* workspace, size_t workspace_bytes,
                                                  void* stream);

/* The NVFP4 operand of x^T: x is the same bf16 [rows, K] matrix as for
 * nvfp4_quantize, but the 16-element blocks run along rows (down a column of
 * x), so codes/scales describe the [K, rows] matrix x^T -- the layout the
 * weight-gradient and input-gradient GEMMs of training need (the "Four Over
 * Six (4/6)" summary, "주요 기여 및 결과": 4/6 applied to weights, activations
 * and gradients in NVFP4 pretraining).  Same alpha (the tensor amax is the
 * same), same modes, rules and arithmetic per block as nvfp4_quantize.
 *   codes   [K, rows/2] bytes, nvfp4_codes_bytes(K, rows)
 *   scales  nvfp4_scales_bytes(K, rows) bytes, swizzled for a [K, rows] operand
 * Requirements: rows a positive multiple of 64, K a positive multiple of 8,
 * ldx >= K and ldx % 8 == 0, buffers as nvfp4_quantize, workspace of
 * nvfp4_quantize_workspace_bytes(rows, K).  Two kernel launches (amax pass,
 * tiled transpose-quantize). */
NVFP4_API nvfp4_status nvfp4_quantize_t(const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                                        int rule, float fp8_max, void* codes, void* scales,
                                        float* global_scale, void* workspace, size_t workspace_bytes,
                                        void* stream);

/* nvfp4_quantize with a caller-supplied tensor scale: alpha is read from
 * *global_scale (device memory; e.g. calibrated offline, or a previous call's
 * output), the tensor-amax pass and its read of x are skipped, and every
 * block is quantized against that alpha (block scales saturate at 448 and
 * codes at 6 where alpha is smaller than amax / (fp8_max * 6)).  Source: the
 * Minima page, "심층 분석" (calibrated module-level scales) -- the quantity is
 * the same alpha the "Four Over Six (4/6)" summary defines in "구현 세부 사항".
 * Same arguments, requirements and outputs as nvfp4_quantize except that
 * fp8_max is not needed and *global_scale is read, not written; the workspace
 * needs only nvfp4_gemm_workspace_bytes() bytes (the status word).  Device
 * status: NVFP4_ERR_INVALID_ARG when alpha is not a positive finite number
 * (nothing written), NVFP4_ERR_NONFINITE when a block holds Inf or NaN (that
 * block's codes and scale are written as zeros).  One 8-byte memset of the
 * status word, then one kernel launch. */
NVFP4_API nvfp4_status nvfp4_quantize_with_scale(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                                 int mode, int rule, const float* global_scale,
                                                 void* codes, void* scales, void* workspace,
                                                 size_t workspace_bytes, void* stream);

/* nvfp4_quantize without a workspace, for callers that cannot allocate device
 * memory where they quantize: a custom-op or plugin hook inside another
 * inference runtime that owns every device allocation and passes the op only
 * its inputs and outputs, or a service whose device-memory footprint is fixed
 * at start-up and which must not allocate on the request path.  The paper has
 * no counterpart; this is an interface convenience of this library.
 * Same arguments, requirements and outputs as nvfp4_quantize, minus the
 * workspace.  The scratch (status word and amax partial maxima) is a static
 * device array of 16448 bytes inside this library, held on every GPU that
 * loads it until the process exits; a launch whose amax pass would need more
 * than its 4096 partial slots is rejected with NVFP4_ERR_INVALID_ARG (a B200
 * uses at most 296, two per SM).  Nothing in the scratch has to start at zero: every call
 * writes what it later reads.  All calls on a device share the array, so calls
 * that may overlap on the GPU race and must be ordered by the caller (same
 * stream, or events).  The first call on each device looks up the array's
 * device address with cudaGetSymbolAddress (with that device current); make
 * that first call before any stream capture.  The array belongs to the CUDA
 * context that loaded this library's module: the lookup is repeated on the
 * first call in every other context of the device (a driver-API context, or
 * the primary context after cudaDeviceReset re-created it), and that call
 * too should come before any stream capture.  Non-finite input shows as a NaN
 * *global_scale (there is no workspace status word to read).  Allocates
 * nothing: no cudaMalloc, cudaFree or allocating library routine. */
NVFP4_API nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                              int mode, int rule, float fp8_max, void* codes,
                                              void* scales, float* global_scale, void* stream);

/* Y [M, N] = (alpha_A * alpha_B) * (A_hat . B_hat^T) with an fp32 accumulator.
 *   a_codes/a_scales/a_global  operand A (M rows), as nvfp4_quantize wrote it
 *   b_codes/b_scales/b_global  operand B (N rows, e.g. a weight [N, K])
 *   out_dtype  NVFP4_OUT_BF16 (round-to-nearest-even) or NVFP4_OUT_FP32.
 * Requirements: 1 <= M, N, K <= 2^30, K % 64 == 0, N <= ldy <= 2^40, code
 * and scale buffers 16-byte aligned, Y aligned to its element size, workspace
 * (>= nvfp4_gemm_workspace_bytes(), 16-byte aligned) for the status word.
 * Enqueues a 64-byte memset of the status word and one kernel launch. */
NVFP4_API nvfp4_status nvfp4_gemm(const void* a_codes, const void* a_scales, const float* a_global,
                        const void* b_codes, const void* b_scales, const float* b_global,
                        int64_t M, int64_t N, int64_t K, void* y, int64_t ldy, int out_dtype,
                        void* workspace, size_t workspace_bytes, void* stream);

/* nvfp4_gemm whose epilogue writes Y as an NVFP4 operand instead of bf16: Y is
 * rounded to bf16 exactly as nvfp4_gemm's bf16 output would be, then each
 * 16-column block goes through the block step of nvfp4_quantize (mode, rule)
 * against the caller-supplied tensor scale *y_alpha (device), so the result
 * equals nvfp4_gemm (bf16) followed by nvfp4_quantize_with_scale, bit for bit,
 * without Y ever being written in bf16.  This is the quantization fused into
 * the producing op's epilogue that a calibrated (static) alpha makes possible
 * (Minima page, "심층 분석": calibrated module-level scales).
 *   y_codes   [M, N/2], 16-byte aligned;  y_scales  nvfp4_scales_bytes(M, N)
 * Requirements as nvfp4_gemm plus N % 64 == 0.  Device status as
 * nvfp4_quantize_with_scale: NVFP4_ERR_INVALID_ARG when *y_alpha is not a
 * positive finite number (nothing is written), NVFP4_ERR_NONFINITE when a
 * block of Y holds Inf/NaN (written as zeros).  One memset, one kernel. */
NVFP4_API nvfp4_status nvfp4_gemm_quantized(const void* a_codes, const void* a_scales, const float* a_global,
                                            const void* b_codes, const void* b_scales, const float* b_global,
                                            int64_t M, int64_t N, int64_t K, int mode, int rule,
                                            const float* y_alpha, void* y_codes, void* y_scales,
                                            void* workspace, size_t workspace_bytes, void* stream);

/* nvfp4_gemm with one B global scale per output-column segment, for one GEMM
 * over several weights fused along N (e.g. the Q, K and V projections, or
 * gate and up), each quantized with its own tensor scale -- for instance
 * module-level calibrated scales.  Column n of Y belongs to the segment s with
 * seg_ends[s-1] <= n < seg_ends[s] (seg_ends[-1] = 0) and is scaled by
 * alpha_A * b_globals[s].  Source: the Minima page, "심층 분석" (the global
 * scale mismatch met when module-level calibrated checkpoints are fused into
 * one GEMM kernel).
 *   b_globals  device array of nseg floats
 *   seg_ends   host array of nseg exclusive end columns, strictly ascending,
 *              each a multiple of 64 except the last, which must equal N
 *   nseg       1 .. 16
 * Everything else as nvfp4_gemm (B's codes and scales are the fused [N, K]
 * operand; when its segments are quantized separately with nvfp4_quantize
 * into one buffer, their row counts must be multiples of 128 so their scale
 * atoms do not overlap).  nseg == 1 with seg_ends = {N} is nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_gemm_segmented(const void* a_codes, const void* a_scales,
                                            const float* a_global, const void* b_codes,
                                            const void* b_scales, const float* b_globals,
                                            const int64_t* seg_ends, int nseg, int64_t M, int64_t N,
                                            int64_t K, void* y, int64_t ldy, int out_dtype,
                                            void* workspace, size_t workspace_bytes, void* stream);

/* The W4A4 linear layer in one call: quantize the activations x [M, K] as
 * nvfp4_quantize does (into x_codes / x_scales / *x_global_scale, with
 * x_workspace), then Y [M, N] = X_hat . W_hat^T as nvfp4_gemm does, against
 * a weight already quantized (w_codes / w_scales / w_global, N rows).  The
 * long-prefill path of the Minima page ("산업 영향"): quantize -> GEMM on one
 * stream.  Enqueues the GEMM's 64-byte status reset, the amax pass, the
 * quantize kernel and the GEMM kernel, each kernel a programmatic dependent
 * of the one before it (it is scheduled while that one drains and waits for
 * it before touching memory), so the quantizer's and the GEMM's prologues
 * overlap the preceding kernel's tail.  Results are those of the two calls
 * made one after the other, bit for bit.  Arguments and requirements are
 * those of nvfp4_quantize and nvfp4_gemm; every one is checked before
 * anything is enqueued.  Device status: x_workspace as nvfp4_quantize,
 * workspace as nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_quantize_gemm(const void* x, int64_t M, int64_t K, int64_t ldx, int mode, int rule,
                                           float fp8_max, void* x_codes, void* x_scales, float* x_global_scale,
                                           void* x_workspace, size_t x_workspace_bytes, const void* w_codes,
                                           const void* w_scales, const float* w_global, int64_t N, void* y,
                                           int64_t ldy, int out_dtype, void* workspace, size_t workspace_bytes,
                                           void* stream);

/* The augmented-channel W4A4 linear layer in one call (ARCQuant page, "방법론":
 * reorder + dual quantization, then one NVFP4 GEMM over K + S): quantize x
 * [M, K] as nvfp4_quantize_arc does with augment = 0 (into x_codes
 * [M, (K+S)/2], x_scales nvfp4_scales_bytes(M, K + S), *x_global_scale, with
 * x_workspace of nvfp4_quantize_workspace_bytes(M, K)), then
 * Y [M, N] = X_aug . W_aug^T as nvfp4_gemm does over K + S, against a weight
 * already quantized by nvfp4_quantize_arc with the same perm and S and
 * augment = 1 (w_codes / w_scales / w_global, N rows, K + S columns).
 * Enqueues the GEMM's status reset, the amax pass, the augmented quantize
 * kernel and the GEMM kernel, each kernel a programmatic dependent of the one
 * before it.  Results are those of the two calls made one after the other, bit
 * for bit.  Arguments and requirements are those of nvfp4_quantize_arc and
 * nvfp4_gemm (with K + S for the GEMM); every one is checked before anything
 * is enqueued.  Device status: x_workspace as nvfp4_quantize_arc, workspace as
 * nvfp4_gemm. */
NVFP4_API nvfp4_status nvfp4_quantize_arc_gemm(const void* x, int64_t M, int64_t K, int64_t ldx,
                                               const int32_t* perm, int64_t S, int mode, int rule, float fp8_max,
                                               void* x_codes, void* x_scales, float* x_global_scale,
                                               void* x_workspace, size_t x_workspace_bytes, const void* w_codes,
                                               const void* w_scales, const float* w_global, int64_t N, void* y,
                                               int64_t ldy, int out_dtype, void* workspace,
                                               size_t workspace_bytes, void* stream);

/* nvfp4_quantize_arc_gemm with the activations' RMSNorm fused ahead: x is
 * quantized as nvfp4_quantize_arc_rmsnorm does (gamma, eps; x_workspace of
 * nvfp4_quantize_arc_rmsnorm_workspace_bytes(M, K)), then the GEMM over K + S
 * against the weight quantized by nvfp4_quantize_arc with the same perm and S
 * and augment = 1.  Results are those of the two calls made one after the
 * other, bit for bit; every argument is checked before anything is enqueued. */
NVFP4_API nvfp4_status nvfp4_quantize_arc_rmsnorm_gemm(const void* x, int64_t M, int64_t K, int64_t ldx,
                                                       const void* gamma, float eps, const int32_t* perm,
                                                       int64_t S, int mode, int rule, float fp8_max,
                                                       void* x_codes, void* x_scales, float* x_global_scale,
                                                       void* x_workspace, size_t x_workspace_bytes,
                                                       const void* w_codes, const void* w_scales,
                                                       const float* w_global, int64_t N, void* y, int64_t ldy,
                                                       int out_dtype, void* workspace, size_t workspace_bytes,
                                                       void* stream);

/* Synchronizes `stream`, then returns the status word the last call that used
 * `workspace` wrote (NVFP4_OK, NVFP4_ERR_INVALID_ARG, NVFP4_ERR_NONFINITE or
 * NVFP4_ERR_TIMEOUT), or
 * NVFP4_ERR_CUDA if the synchronization or the read failed. */
NVFP4_API nvfp4_status nvfp4_get_device_status(const void* workspace, void* stream);

/* Static text for a status code. */
NVFP4_API const char* nvfp4_status_string(nvfp4_status status);

/* Text of the last NVFP4_ERR_CUDA / NVFP4_ERR_INVALID_ARG on this host
 * thread (empty string when none); valid until the next call on the thread. */
NVFP4_API const char* nvfp4_last_error_message(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H */
