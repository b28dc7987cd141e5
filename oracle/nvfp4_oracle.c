/*
 * nvfp4_oracle.c -- plain, slow, scalar CPU definition of NVFP4 quantization
 * (scale-to-6 and Four-Over-Six) used as TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package's smoke check and the benchmark's CPU
 * baseline may load this library.  The product path (the CUDA library under
 * w4a4_gemm_nvfp4_b200/) shares no code, header, table or constant with it.
 *
 * Sources (the pages this build is defined from):
 *   [4/6]  "Four Over Six (4/6)" technical summary, gist.science/ko/paper/2512.02010
 *          - section "문제 제기" (problem statement): E2M1 magnitudes with steps
 *            0.5 on [0,2], 1 on [2,4], 2 on [4,6]; range [-6,6]; under scale-6
 *            the code value 4 sits at 66.6 % of the block maximum.
 *          - section "핵심 메커니즘" (core mechanism): scale-4 maps a block to
 *            [-4,4]; a value at 75 % of the block maximum is exactly 3.
 *          - section "적응형 블록 스케일링 알고리즘" (adaptive block scaling):
 *            quantize every block twice (scale 6 and scale 4), measure each
 *            against the original high-precision values, keep the smaller
 *            error under one of three rules: max error, MAE, MSE.
 *          - section "구현 세부 사항" (implementation details): FP8 E4M3 block
 *            scales; the tensor scale alpha uses FP8 max 256 instead of 448 so
 *            the 1.5x larger scale-4 factor does not overflow E4M3.
 *   [ARC]  "ARCQuant" technical summary, gist.science/ko/paper/2601.07475,
 *          section "문제 정의" (problem definition): NVFP4 blocks are 16
 *          elements along the reduction dimension.
 *
 * Readings where the pages are silent:
 *   - alpha = amax / (F * 6) with F = fp8_max in {448, 256}; alpha = 1 when
 *     amax == 0; a non-finite amax is an error.
 *   - every step is one IEEE-754 binary32 operation, round-to-nearest-even,
 *     in exactly the order written below; no contraction except the one
 *     explicit fmaf() in the error term.
 *   - block scale s = E4M3_RNE_satfinite(b / (alpha * Q)); d = s * alpha;
 *     r = 1 / d, replaced by 0 when that reciprocal is infinite (d == 0 or
 *     d so small that 1/d overflows); elements are scaled by v = x * r.
 *   - element code = E2M1_RNE_satfinite(v): nearest grid value, ties to the
 *     even code, |v| >= 6 -> 6, the sign bit always kept (so -0.1 -> 0x8).
 *   - error e = fmaf(-val(q), d, x) in original units; MAX rule uses max|e|,
 *     MAE uses sum|e|, MSE uses sum(e*e); sums of the 16 terms follow the
 *     contiguous pairwise tree ((t0+t1)+(t2+t3))+... ; pick scale 4 only if its
 *     error is strictly smaller (ties keep scale 6).
 *   - codes: row-major [rows, K/2] bytes, element 2j in the low nibble.
 *   - scales: canonical row-major [rows, K/16] E4M3 bytes; the swizzled copy
 *     used by the block-scaled MMA is 128-row x 4-column atoms of 512 bytes,
 *     byte (r%32)*16 + ((r/32)%4)*4 + (k16%4) inside atom
 *     (r/128) * (K/64) + (k16/4); padding bytes are 0.
 *
 * Compiled with: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -shared -fPIC
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_MODE_SIX 0
#define OR_MODE_FOUR_OVER_SIX 1
#define OR_RULE_MAX 0
#define OR_RULE_MAE 1
#define OR_RULE_MSE 2

/* ---------------------------------------------------------------- E2M1 --- */

/* Magnitudes of the eight non-negative E2M1 codes ([4/6] "문제 제기"):
 * 0, 0.5, 1, 1.5 (step 0.5), 2, 3 (step 1), 4, 6 (step 2). */
static const float kE2M1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float or_e2m1_value(uint8_t code) {
  float m = kE2M1Mag[code & 7u];
  return (code & 8u) ? -m : m;
}

/* Round to the nearest E2M1 value, ties to the even code, saturating at 6.
 * Works on the magnitude and keeps the sign bit of v in bit 3.  Each
 * midpoint between neighbouring grid values (0.25, 0.75, 1.25, 1.75, 2.5,
 * 3.5, 5) is exact in binary32, so the comparisons below are exact. */
uint8_t or_e2m1_encode(float v) {
  uint8_t sign = signbit(v) ? 8u : 0u;
  float a = fabsf(v);
  if (isnan(a)) return (uint8_t)(sign | 7u);
  for (uint8_t c = 0; c < 7; ++c) {
    float mid = (kE2M1Mag[c] + kE2M1Mag[c + 1]) * 0.5f;
    if (a < mid) return (uint8_t)(sign | c);
    if (a == mid) return (uint8_t)(sign | ((c % 2u == 0u) ? c : c + 1u));
  }
  return (uint8_t)(sign | 7u);
}

/* ---------------------------------------------------------------- E4M3 --- */

/* Value of an E4M3 code (bias 7, 3 mantissa bits, subnormals 2^-9 * m,
 * exponent field 15 with mantissa 7 is NaN, no infinities). */
float or_e4m3_value(uint8_t code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  float v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexpf((float)m, -9);
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* Round a non-negative binary32 to E4M3: nearest of the 127 finite
 * non-negative codes (their values increase with the code), ties to the even
 * mantissa (= even code), values above the largest midpoint saturate to 448
 * (code 0x7E).  Midpoints of neighbouring codes have at most 5 significant
 * bits, so they and the comparisons are exact.  NaN maps to 0x7F (never
 * produced for the finite inputs this oracle feeds it). */
uint8_t or_e4m3_encode_satfinite(float v) {
  if (isnan(v)) return 0x7F;
  if (!(v > 0.0f)) return 0;     /* scales are magnitudes: b >= 0, alpha > 0 */
  for (uint8_t c = 0; c < 0x7E; ++c) {
    float mid = (or_e4m3_value(c) + or_e4m3_value((uint8_t)(c + 1))) * 0.5f;
    if (v < mid) return c;
    if (v == mid) return (c % 2u == 0u) ? c : (uint8_t)(c + 1u);
  }
  return 0x7E;
}

/* ---------------------------------------------------------- tensor scale --- */

static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* amax = max |x| over a [rows, K] bf16 tensor with row stride ldx elements.
 * Sets *nonfinite when any element is Inf or NaN. */
float or_amax_bf16(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, int* nonfinite) {
  float amax = 0.0f;
  int bad = 0;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* row = x + r * ldx;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(row[k]));
      if (!isfinite(a)) bad = 1;
      else if (a > amax) amax = a;
    }
  }
  if (nonfinite) *nonfinite = bad;
  return amax;
}

/* alpha = amax / (F * 6): F*6 is 2688 or 1536, exact in binary32; one IEEE
 * division.  An all-zero tensor takes alpha = 1 (reading). */
float or_global_scale(float amax, float fp8_max) {
  float denom = fp8_max * 6.0f;
  if (amax == 0.0f) return 1.0f;
  return amax / denom;
}

/* ------------------------------------------------------------ one block --- */

/* The 16-term contiguous pairwise tree: (t0+t1),(t2+t3),... then pairs of
 * those, and so on, down to one value. */
static float pairwise_sum16(const float t[16]) {
  float a[16];
  memcpy(a, t, sizeof(a));
  for (int n = 16; n > 1; n /= 2)
    for (int i = 0; i < n / 2; ++i) a[i] = a[2 * i] + a[2 * i + 1];
  return a[0];
}

static float block_error(const float e[16], int rule) {
  float t[16];
  if (rule == OR_RULE_MAX) {
    float m = 0.0f;
    for (int i = 0; i < 16; ++i) { float a = fabsf(e[i]); if (a > m) m = a; }
    return m;
  }
  for (int i = 0; i < 16; ++i) t[i] = (rule == OR_RULE_MSE) ? e[i] * e[i] : fabsf(e[i]);
  return pairwise_sum16(t);
}

/* Quantize one 16-element block against scale target Q (6 or 4). */
static void quantize_candidate(const float x[16], float b, float alpha, float Q, int rule,
                               uint8_t codes[16], uint8_t* scale, float* err) {
  float aq = alpha * Q;
  float s_raw = b / aq;
  uint8_t s = or_e4m3_encode_satfinite(s_raw);
  float d = or_e4m3_value(s) * alpha;
  float r = 1.0f / d;
  if (isinf(r)) r = 0.0f;
  float e[16];
  for (int i = 0; i < 16; ++i) {
    float v = x[i] * r;
    codes[i] = or_e2m1_encode(v);
    e[i] = fmaf(-or_e2m1_value(codes[i]), d, x[i]);
  }
  *scale = s;
  *err = block_error(e, rule);
}

/* One candidate on its own (test access): Q = 6 or 4. */
void or_quantize_candidate(const float x[16], float alpha, float Q, int rule, uint8_t codes[16],
                           uint8_t* scale, float* err) {
  float b = 0.0f;
  for (int i = 0; i < 16; ++i) { float a = fabsf(x[i]); if (a > b) b = a; }
  quantize_candidate(x, b, alpha, Q, rule, codes, scale, err);
}

/* Quantize one block.  Outputs the chosen 16 codes (one per byte), the chosen
 * E4M3 scale, and for testing the two candidate errors and the choice
 * (chose4 = 1 when scale 4 was kept; err4 = NAN in mode six). */
void or_quantize_block(const float x[16], float alpha, int mode, int rule,
                       uint8_t codes[16], uint8_t* scale, int* chose4, float* err6, float* err4) {
  float b = 0.0f;
  for (int i = 0; i < 16; ++i) { float a = fabsf(x[i]); if (a > b) b = a; }
  uint8_t c6[16], c4[16], s6, s4;
  float e6, e4 = NAN;
  quantize_candidate(x, b, alpha, 6.0f, rule, c6, &s6, &e6);
  int pick4 = 0;
  if (mode == OR_MODE_FOUR_OVER_SIX) {
    quantize_candidate(x, b, alpha, 4.0f, rule, c4, &s4, &e4);
    pick4 = (e4 < e6);
  }
  memcpy(codes, pick4 ? c4 : c6, 16);
  *scale = pick4 ? s4 : s6;
  if (chose4) *chose4 = pick4;
  if (err6) *err6 = e6;
  if (err4) *err4 = e4;
}

/* -------------------------------------------- augmented residual channels --- */

/* ARCQuant (ARCQuant page, 기술 요약 / 방법론): the activation's K channels are
 * reordered by a calibration permutation (outliers first); the primary stage is
 * the usual NVFP4 quantization of the reordered row; the residual stage takes
 * the first S reordered channels, forms their residual against the primary
 * stage, e_j = fmaf(-val(q_j), d, x_j) with d = val(s)*alpha of the block, and
 * quantizes it as S more NVFP4 channels (same alpha, mode and rule) appended
 * along K, so one GEMM over K + S adds the correction.  augment == 1 instead
 * appends a plain copy of the first S reordered channels (the matching weight
 * columns are duplicated).  Output per row: K + S channels; codes packed
 * [rows, (K+S)/2], canonical scales [rows, (K+S)/16].  Returns 0, or 1 when x
 * holds a non-finite value (outputs untouched). */
int or_quantize_arc(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, const int32_t* perm,
                    int64_t S, int augment, int mode, int rule, float fp8_max, uint8_t* codes,
                    uint8_t* scales, float* alpha_out) {
  int bad = 0;
  float amax = or_amax_bf16(x, rows, K, ldx, &bad);
  if (bad) return 1;
  float alpha = or_global_scale(amax, fp8_max);
  const int64_t KA = K + S;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t j = 0; j < K / 16; ++j) {
      float xb[16];
      uint8_t q[16], s;
      for (int i = 0; i < 16; ++i) xb[i] = bf16_to_f32(x[r * ldx + perm[j * 16 + i]]);
      or_quantize_block(xb, alpha, mode, rule, q, &s, 0, 0, 0);
      scales[r * (KA / 16) + j] = s;
      for (int i = 0; i < 8; ++i)
        codes[r * (KA / 2) + j * 8 + i] = (uint8_t)((q[2 * i] & 15u) | ((q[2 * i + 1] & 15u) << 4));
      if (j * 16 >= S) continue;
      /* the block's augmented channels K + 16j .. K + 16j + 15 */
      const int64_t ja = K / 16 + j;
      uint8_t qa[16], sa;
      if (augment == 1) {
        memcpy(qa, q, 16);
        sa = s;
      } else {
        float e[16];
        const float d = or_e4m3_value(s) * alpha;
        for (int i = 0; i < 16; ++i) e[i] = fmaf(-or_e2m1_value(q[i]), d, xb[i]);
        or_quantize_block(e, alpha, mode, rule, qa, &sa, 0, 0, 0);
      }
      scales[r * (KA / 16) + ja] = sa;
      for (int i = 0; i < 8; ++i)
        codes[r * (KA / 2) + ja * 8 + i] = (uint8_t)((qa[2 * i] & 15u) | ((qa[2 * i + 1] & 15u) << 4));
    }
  }
  if (alpha_out) *alpha_out = alpha;
  return 0;
}

/* ------------------------------------------------------------- RMSNorm --- */

/* Round a binary32 to bf16: nearest, ties to the even bf16 significand;
 * values past the bf16 range round to infinity; a NaN stays a (quiet) NaN.
 * Adding 0x7FFF plus the last kept bit to the bit pattern and truncating is
 * exactly that rounding on the magnitude (the carry moves into the exponent
 * when the significand overflows). */
uint16_t or_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if (isnan(f)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* The contiguous pairwise tree over n terms, padded with zeros to the next
 * power of two (adding +0 changes no partial sum): (t0+t1),(t2+t3),... then
 * pairs of those, down to one value. */
static float pairwise_sum(const float* t, int64_t n) {
  int64_t p = 1;
  while (p < n) p *= 2;
  float* a = (float*)calloc((size_t)p, sizeof(float));
  if (!a) return NAN;
  memcpy(a, t, (size_t)n * sizeof(float));
  for (int64_t m = p; m > 1; m /= 2)
    for (int64_t i = 0; i < m / 2; ++i) a[i] = a[2 * i] + a[2 * i + 1];
  const float sum = a[0];
  free(a);
  return sum;
}

/* RMSNorm of each row of a bf16 [rows, K] tensor with a bf16 gain gamma[K]
 * ([ARC] "방법론", 커널 구현: the fused kernel normalizes the activations before
 * reordering and quantizing them; the page gives no formula, so this is the
 * standard RMSNorm):
 *   ms = (sum_k x_k * x_k) / K    squares exact for finite bf16; the sum
 *                                 is the contiguous pairwise tree; one IEEE
 *                                 division by K
 *   r  = 1 / sqrt(ms + eps)       an IEEE add, a correctly rounded square
 *                                 root, then an IEEE division
 *   y_k = bf16((x_k * r) * gamma_k)  two binary32 products, in that order,
 *                                 rounded to bf16 (the normalized activation
 *                                 is a bf16 tensor, as the quantizer input is)
 * y is [rows, K] contiguous.  Returns 0 (eps is the caller's; a zero row with
 * eps = 0 gives r = inf and NaN outputs). */
int or_rmsnorm_bf16(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, const uint16_t* gamma,
                    float eps, uint16_t* y) {
  float* t = (float*)malloc((size_t)K * sizeof(float));
  if (!t) return 1;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* row = x + r * ldx;
    for (int64_t k = 0; k < K; ++k) {
      const float v = bf16_to_f32(row[k]);
      t[k] = v * v;
    }
    const float ms = pairwise_sum(t, K) / (float)K;
    const float q = sqrtf(ms + eps);
    const float rinv = 1.0f / q;
    for (int64_t k = 0; k < K; ++k) {
      const float xr = bf16_to_f32(row[k]) * rinv;
      y[r * K + k] = or_f32_to_bf16(xr * bf16_to_f32(gamma[k]));
    }
  }
  free(t);
  return 0;
}

/* ------------------------------------------------------------ a tensor --- */

/* Quantize rows of a bf16 tensor with a given alpha.  codes: [nrows, K/2]
 * packed (element 2j low nibble); scales: canonical [nrows, K/16]. */
void or_quantize_rows(const uint16_t* x, int64_t nrows, int64_t K, int64_t ldx, float alpha,
                      int mode, int rule, uint8_t* codes, uint8_t* scales) {
  for (int64_t r = 0; r < nrows; ++r) {
    for (int64_t j = 0; j < K / 16; ++j) {
      float xb[16];
      uint8_t q[16];
      for (int i = 0; i < 16; ++i) xb[i] = bf16_to_f32(x[r * ldx + j * 16 + i]);
      or_quantize_block(xb, alpha, mode, rule, q, &scales[r * (K / 16) + j], 0, 0, 0);
      for (int i = 0; i < 8; ++i)
        codes[r * (K / 2) + j * 8 + i] = (uint8_t)((q[2 * i] & 15u) | ((q[2 * i + 1] & 15u) << 4));
    }
  }
}

/* Whole-tensor quantization: amax -> alpha -> every block.  Returns 0 on
 * success, 1 when the tensor holds a non-finite value (outputs untouched). */
int or_quantize(const uint16_t* x, int64_t rows, int64_t K, int64_t ldx, int mode, int rule,
                float fp8_max, uint8_t* codes, uint8_t* scales, float* alpha_out) {
  int bad = 0;
  float amax = or_amax_bf16(x, rows, K, ldx, &bad);
  if (bad) return 1;
  float alpha = or_global_scale(amax, fp8_max);
  or_quantize_rows(x, rows, K, ldx, alpha, mode, rule, codes, scales);
  if (alpha_out) *alpha_out = alpha;
  return 0;
}

/* ------------------------------------------------------- scale layout ----- */

int64_t or_scales_swizzled_bytes(int64_t rows, int64_t K) {
  return ((rows + 127) / 128) * 128 * (K / 16);
}

/* Canonical [rows, K/16] -> swizzled atoms (buffer of
 * or_scales_swizzled_bytes bytes, padding written as 0).  K % 64 == 0. */
void or_swizzle_scales(const uint8_t* canon, int64_t rows, int64_t K, uint8_t* swz) {
  int64_t kb = K / 16, kgroups = K / 64;
  memset(swz, 0, (size_t)or_scales_swizzled_bytes(rows, K));
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < kb; ++j) {
      int64_t atom = (r / 128) * kgroups + (j / 4);
      int64_t off = (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
      swz[atom * 512 + off] = canon[r * kb + j];
    }
}

/* Swizzled -> canonical (inverse of the above on the first rows rows). */
void or_unswizzle_scales(const uint8_t* swz, int64_t rows, int64_t K, uint8_t* canon) {
  int64_t kb = K / 16, kgroups = K / 64;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t j = 0; j < kb; ++j) {
      int64_t atom = (r / 128) * kgroups + (j / 4);
      int64_t off = (r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);
      canon[r * kb + j] = swz[atom * 512 + off];
    }
}

/* ------------------------------------------------------------ dequant ---- */

/* x_hat[r,k] = val(code) * val(scale) * alpha in binary64 (exact: 2 + 4 + 24
 * significant bits).  codes packed [rows, K/2]; scales canonical [rows, K/16]. */
void or_dequantize(const uint8_t* codes, const uint8_t* scales, float alpha, int64_t rows,
                   int64_t K, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = codes[r * (K / 2) + k / 2];
      uint8_t c = (k % 2) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
      double s = (double)or_e4m3_value(scales[r * (K / 16) + k / 16]);
      out[r * K + k] = (double)or_e2m1_value(c) * s * (double)alpha;
    }
}
