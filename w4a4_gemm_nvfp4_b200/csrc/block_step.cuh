// block_step.cuh -- the NVFP4 block step shared by the quantizer kernels and
// the GEMM epilogue that writes a quantized output.
//
// Definition ("Four Over Six (4/6)" technical summary,
// gist.science/ko/paper/2512.02010; sections "문제 제기", "적응형 블록 스케일링
// 알고리즘", "구현 세부 사항"):
//   per 16-element block, b = max|x|; for Q in {6} or {6, 4}:
//     s = E4M3_RNE_satfinite(b / (alpha*Q)), d = s*alpha, r = 1/d (0 if inf)
//     q_i = E2M1_RNE_satfinite(x_i * r), e_i = fma(-q_i, d, x_i)
//     E_Q = max|e| | sum|e| | sum e^2 (contiguous pairwise tree)
//   keep Q = 4 iff E_4 < E_6.
// Every step is one binary32 operation (explicit __f*_rn intrinsics and
// packed f32x2 PTX), so the result does not depend on FMA contraction.
#pragma once

#include <cstdint>

namespace nvfp4 {
namespace {

constexpr uint32_t kAbsMask2 = 0x7FFF7FFFu;  // clears both bf16 sign bits

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t absmax4(const uint4& v, uint32_t m) {
  m = max_u16x2(m, v.x & kAbsMask2);
  m = max_u16x2(m, v.y & kAbsMask2);
  m = max_u16x2(m, v.z & kAbsMask2);
  return max_u16x2(m, v.w & kAbsMask2);
}

// Three-input maximum that propagates NaN (one instruction on sm_100; the
// compiler folds fabsf of an operand into it).
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
  float d;
  asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ------------------------------------------------------- conversions ----

// Two binary32 -> two E4M3 (RNE, saturating to 448): lo byte from `lo`.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}
// Two E4M3 (byte pair) -> two binary32 (exact, via f16).
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t pair, float& lo, float& hi) {
  asm("{\n\t.reg .b32 h2;\n\t.reg .f16 h0, h1;\n\t"
      "cvt.rn.f16x2.e4m3x2 h2, %2;\n\t"
      "mov.b32 {h0, h1}, h2;\n\t"
      "cvt.f32.f16 %0, h0;\n\t"
      "cvt.f32.f16 %1, h1;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "h"(static_cast<uint16_t>(pair)));
}
// Two binary32 -> E2M1 codes (RNE, saturating to 6, sign kept); the code byte
// holds `lo` in its low nibble.
__device__ __forceinline__ uint32_t e2m1x2_encode(float hi, float lo) {
  uint32_t byte;
  asm("{\n\t.reg .b8 c;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 c, %1, %2;\n\t"
      "cvt.u32.u8 %0, c;\n\t}"
      : "=r"(byte)
      : "f"(hi), "f"(lo));
  return byte;
}
// Packed binary32 pairs held in one 64-bit register pair (one IEEE RNE
// operation per lane, like the scalar instruction on each lane).
struct f2 {
  uint64_t v;
  __device__ __forceinline__ float a() const { return __uint_as_float(static_cast<uint32_t>(v)); }
  __device__ __forceinline__ float b() const { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
};
__device__ __forceinline__ f2 make_f2(float a, float b) {
  f2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r.v) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ f2 mul2(f2 x, f2 y) {
  f2 r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(x.v), "l"(y.v));
  return r;
}
__device__ __forceinline__ f2 fma2(f2 x, f2 y, f2 z) {
  f2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.v) : "l"(x.v), "l"(y.v), "l"(z.v));
  return r;
}
__device__ __forceinline__ f2 add2(f2 x, f2 y) {
  f2 r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r.v) : "l"(x.v), "l"(y.v));
  return r;
}

__device__ __forceinline__ float safe_recip(float d) {
  float r = __frcp_rn(d);
  return isinf(r) ? 0.0f : r;  // d == 0 or 1/d overflowed
}

enum { kRuleMax = 0, kRuleMae = 1, kRuleMse = 2 };

// The block step's per-scale-code constants, one 16-byte shared-memory entry
// per E4M3 code c: (r, r) and (-d, -d) with d = val(c) * alpha and r = 1/d
// (0 if infinite), already paired for the packed f32x2 arithmetic.
struct __align__(16) ScaleEntry {
  f2 rr;  // (r, r)
  f2 nd;  // (-d, -d)
};
__device__ __forceinline__ void load_entry(const ScaleEntry* tab, uint32_t code, f2& rr, f2& nd) {
  asm("ld.shared.v2.b64 {%0, %1}, [%2];"
      : "=l"(rr.v), "=l"(nd.v)
      : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(tab + code))));
}
__device__ __forceinline__ f2 load_rr(const ScaleEntry* tab, uint32_t code) {
  f2 rr;
  asm("ld.shared.b64 %0, [%1];" : "=l"(rr.v) : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(tab + code))));
  return rr;
}

// Codes of one candidate: v = x * r per element, E2M1-rounded.  The block's
// 16 values are held as pairs p[j] = (x_j, x_{j+8}), j < 8; codes byte j holds
// elements 2j, 2j+1 (low nibble first).
__device__ __forceinline__ uint2 candidate_codes(const f2 p[8], f2 rr) {
  uint32_t bytes[8];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const f2 v0 = mul2(p[2 * j], rr), v1 = mul2(p[2 * j + 1], rr);
    bytes[j] = e2m1x2_encode(v1.a(), v0.a());
    bytes[j + 4] = e2m1x2_encode(v1.b(), v0.b());
  }
  return make_uint2(bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24),
                    bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24));
}

// One candidate with its block error under RULE.  With the (x_j, x_{j+8})
// pairing the contiguous pairwise tree of the error terms
// ((t0+t1)+(t2+t3))+... is exactly three packed additions and one scalar one:
//   (t_2i + t_2i+1, t_2i+8 + t_2i+9)      = (u_i, u_i+4)   i < 4
//   (u_2i + u_2i+1, u_2i+4 + u_2i+5)      = (w_i, w_i+2)   i < 2
//   (w_0 + w_1, w_2 + w_3)                = (z_0, z_1),    then z_0 + z_1.
// E2M1 encode of v (pairs v[j] = (v_j, v_{j+8})) into the two code words
// (element i in nibble i of codes.x for i < 8, of codes.y for i >= 8; RNE,
// saturating to 6, sign kept) and the code values back as binary32 (exact,
// via f16), written directly as the pairs q[j] = (val(code j), val(code
// j+8)) that the packed error arithmetic takes.
__device__ __forceinline__ void encode_decode(const f2 v[8], uint2& codes, f2 q[8]) {
  asm("{\n\t.reg .f32 a<8>, b<8>, qa<8>, qb<8>;\n\t.reg .b8 cx<4>, cy<4>;\n\t"
      ".reg .b32 hx<4>, hy<4>;\n\t.reg .f16 fa<8>, fb<8>;\n\t"
      "mov.b64 {a0, b0}, %10;\n\tmov.b64 {a1, b1}, %11;\n\tmov.b64 {a2, b2}, %12;\n\tmov.b64 {a3, b3}, %13;\n\t"
      "mov.b64 {a4, b4}, %14;\n\tmov.b64 {a5, b5}, %15;\n\tmov.b64 {a6, b6}, %16;\n\tmov.b64 {a7, b7}, %17;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 cx0, a1, a0;\n\tcvt.rn.satfinite.e2m1x2.f32 cx1, a3, a2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 cx2, a5, a4;\n\tcvt.rn.satfinite.e2m1x2.f32 cx3, a7, a6;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 cy0, b1, b0;\n\tcvt.rn.satfinite.e2m1x2.f32 cy1, b3, b2;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 cy2, b5, b4;\n\tcvt.rn.satfinite.e2m1x2.f32 cy3, b7, b6;\n\t"
      "mov.b32 %0, {cx0, cx1, cx2, cx3};\n\tmov.b32 %1, {cy0, cy1, cy2, cy3};\n\t"
      "cvt.rn.f16x2.e2m1x2 hx0, cx0;\n\tcvt.rn.f16x2.e2m1x2 hx1, cx1;\n\t"
      "cvt.rn.f16x2.e2m1x2 hx2, cx2;\n\tcvt.rn.f16x2.e2m1x2 hx3, cx3;\n\t"
      "cvt.rn.f16x2.e2m1x2 hy0, cy0;\n\tcvt.rn.f16x2.e2m1x2 hy1, cy1;\n\t"
      "cvt.rn.f16x2.e2m1x2 hy2, cy2;\n\tcvt.rn.f16x2.e2m1x2 hy3, cy3;\n\t"
      "mov.b32 {fa0, fa1}, hx0;\n\tmov.b32 {fa2, fa3}, hx1;\n\tmov.b32 {fa4, fa5}, hx2;\n\tmov.b32 {fa6, fa7}, hx3;\n\t"
      "mov.b32 {fb0, fb1}, hy0;\n\tmov.b32 {fb2, fb3}, hy1;\n\tmov.b32 {fb4, fb5}, hy2;\n\tmov.b32 {fb6, fb7}, hy3;\n\t"
      "cvt.f32.f16 qa0, fa0;\n\tcvt.f32.f16 qb0, fb0;\n\tmov.b64 %2, {qa0, qb0};\n\t"
      "cvt.f32.f16 qa1, fa1;\n\tcvt.f32.f16 qb1, fb1;\n\tmov.b64 %3, {qa1, qb1};\n\t"
      "cvt.f32.f16 qa2, fa2;\n\tcvt.f32.f16 qb2, fb2;\n\tmov.b64 %4, {qa2, qb2};\n\t"
      "cvt.f32.f16 qa3, fa3;\n\tcvt.f32.f16 qb3, fb3;\n\tmov.b64 %5, {qa3, qb3};\n\t"
      "cvt.f32.f16 qa4, fa4;\n\tcvt.f32.f16 qb4, fb4;\n\tmov.b64 %6, {qa4, qb4};\n\t"
      "cvt.f32.f16 qa5, fa5;\n\tcvt.f32.f16 qb5, fb5;\n\tmov.b64 %7, {qa5, qb5};\n\t"
      "cvt.f32.f16 qa6, fa6;\n\tcvt.f32.f16 qb6, fb6;\n\tmov.b64 %8, {qa6, qb6};\n\t"
      "cvt.f32.f16 qa7, fa7;\n\tcvt.f32.f16 qb7, fb7;\n\tmov.b64 %9, {qa7, qb7};\n\t}"
      : "=r"(codes.x), "=r"(codes.y), "=l"(q[0].v), "=l"(q[1].v), "=l"(q[2].v), "=l"(q[3].v), "=l"(q[4].v),
        "=l"(q[5].v), "=l"(q[6].v), "=l"(q[7].v)
      : "l"(v[0].v), "l"(v[1].v), "l"(v[2].v), "l"(v[3].v), "l"(v[4].v), "l"(v[5].v), "l"(v[6].v), "l"(v[7].v));
}

// One candidate with its block error under RULE.  With the (x_j, x_{j+8})
// pairing the contiguous pairwise tree of the error terms
// ((t0+t1)+(t2+t3))+... is exactly three packed additions and one scalar one:
//   (t_2i + t_2i+1, t_2i+8 + t_2i+9)      = (u_i, u_i+4)   i < 4
//   (u_2i + u_2i+1, u_2i+4 + u_2i+5)      = (w_i, w_i+2)   i < 2
//   (w_0 + w_1, w_2 + w_3)                = (z_0, z_1),    then z_0 + z_1.
template <int RULE>
__device__ __forceinline__ float candidate(const f2 p[8], f2 rr, f2 nd, uint2& codes) {
  f2 v[8], q[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = mul2(p[j], rr);
  encode_decode(v, codes, q);
  // e = fma(-q, d, x), paired like p
  f2 e[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) e[j] = fma2(q[j], nd, p[j]);
  if (RULE == kRuleMax) {
    // max |e| (exact in any order; the errors are finite), one pair at a time
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = max3_nan(m, fabsf(e[j].a()), fabsf(e[j].b()));
    return m;
  }
  f2 t[8];
  if (RULE == kRuleMse) {
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j] = mul2(e[j], e[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) t[j].v = e[j].v & 0x7FFFFFFF7FFFFFFFull;  // |e| of both lanes
  }
  const f2 u0 = add2(t[0], t[1]), u1 = add2(t[2], t[3]), u2 = add2(t[4], t[5]), u3 = add2(t[6], t[7]);
  const f2 w0 = add2(u0, u1), w1 = add2(u2, u3);
  const f2 z = add2(w0, w1);
  return __fadd_rn(z.a(), z.b());
}

// Per-call constants of the block step.  The scale quotient b / (alpha*Q) must
// be the correctly rounded binary32 quotient before its E4M3 rounding; it is
// taken as b * fl(1/(alpha*Q)), which is within 3 units in the last place of
// the quotient, and recomputed by a true division whenever that distance
// could change the E4M3 result: below the E4M3 normal range (2^-6), or with
// the 20 bits under E4M3's 3-bit mantissa within 5 units of the rounding
// midpoint 0x80000.  Above 448 both saturate to 448.
struct BlockConsts {
  float a6, a4;      // alpha * 6, alpha * 4
  float inv6, inv4;  // fl(1 / a6), fl(1 / a4)
  bool fast_div;     // both reciprocals finite and normal
};
__device__ __forceinline__ bool needs_exact_quotient(float q) {
  const uint32_t b = __float_as_uint(q);
  return b < 0x3C800008u || ((b & 0xFFFFFu) - 0x7FFFBu) < 11u;
}

// The block step on 16 binary32 values held as pairs p[j] = (x_j, x_{j+8})
// with block max b: scale(s) and codes of the chosen candidate.  tab[c] holds
// the constants of E4M3 scale code c (ScaleEntry).
template <bool FOUR_OVER_SIX, int RULE>
__device__ __forceinline__ void quantize_pairs(const f2 p[8], float b, const BlockConsts& k,
                                               const ScaleEntry* tab, uint2& codes, uint32_t& scale) {
  float s6raw = __fmul_rn(b, k.inv6);
  float s4raw = FOUR_OVER_SIX ? __fmul_rn(b, k.inv4) : 0.0f;
  if (!k.fast_div || needs_exact_quotient(s6raw) || (FOUR_OVER_SIX && needs_exact_quotient(s4raw))) {
    s6raw = __fdiv_rn(b, k.a6);
    if (FOUR_OVER_SIX) s4raw = __fdiv_rn(b, k.a4);
  }
  const uint32_t sc = cvt_e4m3x2(s4raw, s6raw);  // low byte: scale-6, high byte: scale-4
  if (!FOUR_OVER_SIX) {
    codes = candidate_codes(p, load_rr(tab, sc & 0xFFu));
    scale = sc & 0xFFu;
    return;
  }
  f2 rr6, nd6, rr4, nd4;
  load_entry(tab, sc & 0xFFu, rr6, nd6);
  load_entry(tab, sc >> 8, rr4, nd4);
  uint2 c6, c4;
  const float E6 = candidate<RULE>(p, rr6, nd6, c6);
  const float E4 = candidate<RULE>(p, rr4, nd4, c4);
  const bool pick4 = E4 < E6;  // ties keep scale 6
  codes = pick4 ? c4 : c6;
  scale = pick4 ? (sc >> 8) : (sc & 0xFFu);
}


// bf16 block (8 words of bf16 pairs, element 2j in the low half of word j) ->
// binary32 pairs p[j] = (x_j, x_{j+8}); returns the block's max |x| bit
// pattern (0x7F80 and above: Inf or NaN).
__device__ __forceinline__ uint32_t unpack_block(const uint4& lo, const uint4& hi, f2 p[8]) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    // bf16 -> binary32 as a mixed-precision add of -0 (exact for every bf16
    // value, signed zeros included), which runs on the FMA pipe instead of
    // taking integer shifts and masks
    // (the pairs are formed inside the asm, so no register moves are needed)
    asm("{\n\t.reg .b16 l0, h0, l1, h1;\n\t.reg .f32 a0, a1, b0, b1;\n\t"
        "mov.b32 {l0, h0}, %2;\n\t"
        "mov.b32 {l1, h1}, %3;\n\t"
        "add.rn.f32.bf16 a0, l0, 0f80000000;\n\t"
        "add.rn.f32.bf16 a1, l1, 0f80000000;\n\t"
        "add.rn.f32.bf16 b0, h0, 0f80000000;\n\t"
        "add.rn.f32.bf16 b1, h1, 0f80000000;\n\t"
        "mov.b64 %0, {a0, a1};\n\t"
        "mov.b64 %1, {b0, b1};\n\t}"
        : "=l"(p[2 * i].v), "=l"(p[2 * i + 1].v)
        : "r"(w[i]), "r"(w[i + 4]));
  }
  // max |x| of the 16 values (exact: a maximum of bf16 values), NaN kept
  const float m0 = max3_nan(fabsf(p[0].a()), fabsf(p[1].a()), fabsf(p[2].a()));
  const float m1 = max3_nan(fabsf(p[3].a()), fabsf(p[4].a()), fabsf(p[5].a()));
  const float m2 = max3_nan(fabsf(p[6].a()), fabsf(p[7].a()), fabsf(p[0].b()));
  const float m3 = max3_nan(fabsf(p[1].b()), fabsf(p[2].b()), fabsf(p[3].b()));
  const float m4 = max3_nan(fabsf(p[4].b()), fabsf(p[5].b()), fabsf(p[6].b()));
  const float m = max3_nan(max3_nan(m0, m1, m2), max3_nan(m3, m4, fabsf(p[7].b())), 0.0f);
  return __float_as_uint(m) >> 16;  // its bf16 bit pattern
}

// Quantize one bf16 block; returns its max |x| bit pattern.
template <bool FOUR_OVER_SIX, int RULE>
__device__ __forceinline__ uint32_t quantize_block(const uint4& lo, const uint4& hi, const BlockConsts& k,
                                                   const ScaleEntry* tab, uint2& codes, uint32_t& scale) {
  f2 p[8];
  const uint32_t bbits = unpack_block(lo, hi, p);
  quantize_pairs<FOUR_OVER_SIX, RULE>(p, __uint_as_float(bbits << 16), k, tab, codes, scale);
  return bbits;
}

// E2M1 codes (element i in nibble i of c.x for i < 8, of c.y for i >= 8) back
// to binary32 pairs q[j] = (val(code j), val(code j+8)), exact via f16.
__device__ __forceinline__ void decode_pairs(const uint2 c, f2 q[8]) {
  asm("{\n\t.reg .f32 qa<8>, qb<8>;\n\t.reg .b8 cx<4>, cy<4>;\n\t"
      ".reg .b32 hx<4>, hy<4>;\n\t.reg .f16 fa<8>, fb<8>;\n\t"
      "mov.b32 {cx0, cx1, cx2, cx3}, %8;\n\tmov.b32 {cy0, cy1, cy2, cy3}, %9;\n\t"
      "cvt.rn.f16x2.e2m1x2 hx0, cx0;\n\tcvt.rn.f16x2.e2m1x2 hx1, cx1;\n\t"
      "cvt.rn.f16x2.e2m1x2 hx2, cx2;\n\tcvt.rn.f16x2.e2m1x2 hx3, cx3;\n\t"
      "cvt.rn.f16x2.e2m1x2 hy0, cy0;\n\tcvt.rn.f16x2.e2m1x2 hy1, cy1;\n\t"
      "cvt.rn.f16x2.e2m1x2 hy2, cy2;\n\tcvt.rn.f16x2.e2m1x2 hy3, cy3;\n\t"
      "mov.b32 {fa0, fa1}, hx0;\n\tmov.b32 {fa2, fa3}, hx1;\n\tmov.b32 {fa4, fa5}, hx2;\n\tmov.b32 {fa6, fa7}, hx3;\n\t"
      "mov.b32 {fb0, fb1}, hy0;\n\tmov.b32 {fb2, fb3}, hy1;\n\tmov.b32 {fb4, fb5}, hy2;\n\tmov.b32 {fb6, fb7}, hy3;\n\t"
      "cvt.f32.f16 qa0, fa0;\n\tcvt.f32.f16 qb0, fb0;\n\tmov.b64 %0, {qa0, qb0};\n\t"
      "cvt.f32.f16 qa1, fa1;\n\tcvt.f32.f16 qb1, fb1;\n\tmov.b64 %1, {qa1, qb1};\n\t"
      "cvt.f32.f16 qa2, fa2;\n\tcvt.f32.f16 qb2, fb2;\n\tmov.b64 %2, {qa2, qb2};\n\t"
      "cvt.f32.f16 qa3, fa3;\n\tcvt.f32.f16 qb3, fb3;\n\tmov.b64 %3, {qa3, qb3};\n\t"
      "cvt.f32.f16 qa4, fa4;\n\tcvt.f32.f16 qb4, fb4;\n\tmov.b64 %4, {qa4, qb4};\n\t"
      "cvt.f32.f16 qa5, fa5;\n\tcvt.f32.f16 qb5, fb5;\n\tmov.b64 %5, {qa5, qb5};\n\t"
      "cvt.f32.f16 qa6, fa6;\n\tcvt.f32.f16 qb6, fb6;\n\tmov.b64 %6, {qa6, qb6};\n\t"
      "cvt.f32.f16 qa7, fa7;\n\tcvt.f32.f16 qb7, fb7;\n\tmov.b64 %7, {qa7, qb7};\n\t}"
      : "=l"(q[0].v), "=l"(q[1].v), "=l"(q[2].v), "=l"(q[3].v), "=l"(q[4].v), "=l"(q[5].v), "=l"(q[6].v),
        "=l"(q[7].v)
      : "r"(c.x), "r"(c.y));
}

// Per-call constants and the table of every E4M3 scale code for a given
// alpha; the table needs 128 threads (thread t fills entry t).
__device__ __forceinline__ void make_block_consts(float alpha, BlockConsts& k) {
  k.a6 = __fmul_rn(alpha, 6.0f);
  k.a4 = __fmul_rn(alpha, 4.0f);
  k.inv6 = __frcp_rn(k.a6);
  k.inv4 = __frcp_rn(k.a4);
  k.fast_div = k.inv6 >= 1.17549435e-38f && !isinf(k.inv4);
}
__device__ __forceinline__ void fill_scale_table(float alpha, ScaleEntry* tab, uint32_t t) {
  if (t < 128) {
    float s, unused;
    e4m3x2_to_f32(t, s, unused);
    const float d = t == 0x7F ? 0.0f : __fmul_rn(s, alpha);  // 0x7F is NaN and never produced
    const float r = safe_recip(d);
    tab[t].rr = make_f2(r, r);
    tab[t].nd = make_f2(-d, -d);
  }
}

}  // namespace
}  // namespace nvfp4
