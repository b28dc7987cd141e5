// quantize.cu -- NVFP4 16-element block quantization, scale-to-6 and
// Four-Over-Six, for sm_100a.
//
// Definition ("Four Over Six (4/6)" technical summary,
// gist.science/ko/paper/2512.02010; sections "문제 제기", "적응형 블록 스케일링
// 알고리즘", "구현 세부 사항"):
//   alpha = amax / (fp8_max * 6)                    (1 when amax == 0)
//   per 16-element block along K, b = max|x|; for Q in {6} or {6, 4}:
//     s = E4M3_RNE_satfinite(b / (alpha*Q)), d = s*alpha, r = 1/d (0 if inf)
//     q_i = E2M1_RNE_satfinite(x_i * r), e_i = fma(-q_i, d, x_i)
//     E_Q = max|e| | sum|e| | sum e^2 (contiguous pairwise tree)
//   keep Q = 4 iff E_4 < E_6.
// Every step is one binary32 operation (explicit __f*_rn intrinsics; the
// file is also built with -fmad=false) so the result is bit-reproducible.
//
// Two kernels per call:
//   amax_kernel      one HBM read of x; each CTA writes the max |bf16| bit
//                    pattern it saw to a partials array in the workspace.
//   quantize_kernel  reduces the partials (a few KB, L2-resident) to alpha in
//                    every CTA, then makes one HBM pass over x: each lane owns
//                    one whole 16-element block (two 16-byte loads), so the
//                    block max and both candidates' errors stay in registers
//                    with no shuffles; a warp's 32 lanes cover 8 rows x 4
//                    blocks chosen so that their 32 scale bytes form one
//                    contiguous 32-byte piece of a 512-byte scale atom, and
//                    their codes form eight 32-byte row segments.
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kAmaxThreads = 256;
constexpr int kMaxPartials = 4096;
constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr uint32_t kAbsMask2 = 0x7FFF7FFFu;  // clears both bf16 sign bits

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t absmax4(const uint4& v, uint32_t m) {
  m = max_u16x2(m, v.x & kAbsMask2);
  m = max_u16x2(m, v.y & kAbsMask2);
  m = max_u16x2(m, v.z & kAbsMask2);
  return max_u16x2(m, v.w & kAbsMask2);
}

// ------------------------------------------------------------- amax pass --
// Magnitudes compare like their bit patterns once the sign is cleared, and
// every NaN pattern (> 0x7F80) compares above Inf (0x7F80) above any finite
// value, so one unsigned max gives both amax and the non-finite flag.
__global__ void __launch_bounds__(kAmaxThreads)
    amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                uint32_t* __restrict__ partials) {
  uint32_t m = 0;
  if (ldx == K) {
    const uint4* v = reinterpret_cast<const uint4*>(x);
    const int64_t n = rows * K / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
      uint4 a = ld_stream(v + i), b = ld_stream(v + i + stride);
      uint4 c = ld_stream(v + i + 2 * stride), d = ld_stream(v + i + 3 * stride);
      m = absmax4(a, m);
      m = absmax4(b, m);
      m = absmax4(c, m);
      m = absmax4(d, m);
    }
    for (; i < n; i += stride) m = absmax4(ld_stream(v + i), m);
  } else {
    const int64_t k8 = K / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
      const uint4* v = reinterpret_cast<const uint4*>(x + r * ldx);
      for (int64_t c = threadIdx.x; c < k8; c += blockDim.x) m = absmax4(ld_stream(v + c), m);
    }
  }
  uint32_t m32 = max(m & 0xFFFFu, m >> 16);
#pragma unroll
  for (int o = 16; o; o >>= 1) m32 = max(m32, __shfl_xor_sync(0xffffffffu, m32, o));
  __shared__ uint32_t s_max[kAmaxThreads / 32];
  if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m32;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = 0;
#pragma unroll
    for (int w = 0; w < kAmaxThreads / 32; ++w) r = max(r, s_max[w]);
    partials[blockIdx.x] = r;
  }
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
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(pair)));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16)));
}
// Two binary32 -> one byte of two E2M1 codes (RNE, saturating to 6, sign kept):
// low nibble from `lo`.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float hi, float lo) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
      "cvt.u32.u8 %0, t;\n\t}"
      : "=r"(r)
      : "f"(hi), "f"(lo));
  return r;
}
// One byte of two E2M1 codes -> the two values as binary32 (exact, via f16).
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi) {
  uint32_t h;
  asm("{\n\t.reg .b8 t;\n\t"
      "cvt.u8.u32 t, %1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
      : "=r"(h)
      : "r"(byte));
  lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFFu)));
  hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h >> 16)));
}

__device__ __forceinline__ float safe_recip(float d) {
  float r = __frcp_rn(d);
  return isinf(r) ? 0.0f : r;  // d == 0 or 1/d overflowed
}

// The 16-term contiguous pairwise tree ((t0+t1)+(t2+t3))+...
__device__ __forceinline__ float pairwise16(float t[16]) {
#pragma unroll
  for (int n = 16; n > 1; n >>= 1) {
#pragma unroll
    for (int i = 0; i < n / 2; ++i) t[i] = __fadd_rn(t[2 * i], t[2 * i + 1]);
  }
  return t[0];
}

enum { kRuleMax = 0, kRuleMae = 1, kRuleMse = 2 };

// One candidate: codes (8 bytes, element 2j in the low nibble of byte j) and
// its block error under RULE.
template <int RULE>
__device__ __forceinline__ float candidate(const float x[16], float d, float r, uint2& codes) {
  float t[16];
  uint32_t bytes[8];
  const float nd = -d;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float v0 = __fmul_rn(x[2 * j], r);
    const float v1 = __fmul_rn(x[2 * j + 1], r);
    bytes[j] = cvt_e2m1x2(v1, v0);
    float q0, q1;
    e2m1x2_to_f32(bytes[j], q0, q1);
    const float e0 = __fmaf_rn(q0, nd, x[2 * j]);
    const float e1 = __fmaf_rn(q1, nd, x[2 * j + 1]);
    if (RULE == kRuleMse) {
      t[2 * j] = __fmul_rn(e0, e0);
      t[2 * j + 1] = __fmul_rn(e1, e1);
    } else {
      t[2 * j] = fabsf(e0);
      t[2 * j + 1] = fabsf(e1);
    }
  }
  codes.x = bytes[0] | (bytes[1] << 8) | (bytes[2] << 16) | (bytes[3] << 24);
  codes.y = bytes[4] | (bytes[5] << 8) | (bytes[6] << 16) | (bytes[7] << 24);
  if (RULE == kRuleMax) {
    float m = t[0];
#pragma unroll
    for (int i = 1; i < 16; ++i) m = fmaxf(m, t[i]);
    return m;
  }
  return pairwise16(t);
}

// Quantize one block held as 8 words of bf16 pairs (element 2j in the low
// half of word j).
template <bool FOUR_OVER_SIX, int RULE>
__device__ __forceinline__ void quantize_block(const uint4& lo, const uint4& hi, float alpha,
                                               float a6, float a4, uint2& codes,
                                               uint32_t& scale) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t m = absmax4(lo, 0u);
  m = absmax4(hi, m);
  const float b = __uint_as_float(max(m & 0xFFFFu, m >> 16) << 16);
  float x[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
  const float s6raw = __fdiv_rn(b, a6);
  const float s4raw = FOUR_OVER_SIX ? __fdiv_rn(b, a4) : 0.0f;
  const uint32_t sc = cvt_e4m3x2(s4raw, s6raw);  // low byte: scale-6, high byte: scale-4
  float s6, s4;
  e4m3x2_to_f32(sc, s6, s4);
  const float d6 = __fmul_rn(s6, alpha);
  uint2 c6;
  const float E6 = candidate<RULE>(x, d6, safe_recip(d6), c6);
  if (!FOUR_OVER_SIX) {
    codes = c6;
    scale = sc & 0xFFu;
    return;
  }
  const float d4 = __fmul_rn(s4, alpha);
  uint2 c4;
  const float E4 = candidate<RULE>(x, d4, safe_recip(d4), c4);
  const bool pick4 = E4 < E6;  // ties keep scale 6
  codes = pick4 ? c4 : c6;
  scale = pick4 ? (sc >> 8) : (sc & 0xFFu);
}

struct QuantParams {
  const uint16_t* x;
  int64_t rows, K, ldx;
  uint8_t* codes;
  uint8_t* scales;
  float* global_scale;
  const uint32_t* partials;
  WorkspaceHeader* ws;
  int nparts;
  float f6;            // fp8_max * 6
  uint32_t ntasks;     // ceil(rows/128) * 16 * (K/64)
  uint32_t kgroups;    // K / 64
};

template <bool FOUR_OVER_SIX, int RULE>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_kernel(const QuantParams p) {
  // ---- tensor amax -> alpha (every CTA reduces the same partials) ----
  __shared__ uint32_t s_red[kQuantWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t m = 0;
  for (int i = threadIdx.x; i < p.nparts; i += kQuantThreads) m = max(m, p.partials[i]);
#pragma unroll
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[warp] = m;
  __syncthreads();
  uint32_t amax_bits = 0;
#pragma unroll
  for (int w = 0; w < kQuantWarps; ++w) amax_bits = max(amax_bits, s_red[w]);
  const bool nonfinite = amax_bits >= 0x7F80u;
  const float alpha =
      amax_bits == 0 ? 1.0f : __fdiv_rn(__uint_as_float(amax_bits << 16), p.f6);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.ws->status = nonfinite ? NVFP4_ERR_NONFINITE : NVFP4_OK;
    p.ws->detail = amax_bits;
    *p.global_scale = nonfinite ? __uint_as_float(0x7FC00000u) : alpha;
  }
  if (nonfinite) return;
  const float a6 = __fmul_rn(alpha, 6.0f);
  const float a4 = __fmul_rn(alpha, 4.0f);

  // ---- lane -> (row, 16-element block) inside a warp task ----
  // task = (row_block * 16 + piece) * kgroups + kgroup; a piece is 32 bytes of
  // a 512-byte scale atom: atom byte o = 32*piece + lane holds the scale of
  // row (o/16) + 32*((o/4)%4) and K-block o%4 of the atom.
  const int row_in_atom = ((lane >> 2) & 3) * 32 + (lane >> 4);
  const int kb_in_group = lane & 3;
  const uint32_t total_warps = gridDim.x * kQuantWarps;
  const int64_t half_k = p.K / 2;
  for (uint32_t task = blockIdx.x * kQuantWarps + warp; task < p.ntasks; task += total_warps) {
    const uint32_t kg = task % p.kgroups;
    const uint32_t t2 = task / p.kgroups;
    const uint32_t piece = t2 & 15u, rb = t2 >> 4;
    const int64_t row = static_cast<int64_t>(rb) * 128 + row_in_atom + 2 * piece;
    const int64_t kb = static_cast<int64_t>(kg) * 4 + kb_in_group;
    uint32_t scale = 0;
    if (row < p.rows) {
      const uint4* src = reinterpret_cast<const uint4*>(p.x + row * p.ldx + kb * 16);
      const uint4 lo = ld_stream(src), hi = ld_stream(src + 1);
      uint2 codes;
      quantize_block<FOUR_OVER_SIX, RULE>(lo, hi, alpha, a6, a4, codes, scale);
      *reinterpret_cast<uint2*>(p.codes + row * half_k + kb * 8) = codes;
    }
    p.scales[(static_cast<int64_t>(rb) * p.kgroups + kg) * 512 + piece * 32 + lane] =
        static_cast<uint8_t>(scale);
  }
}

template <bool F, int R>
cudaError_t launch_quantize(int grid, const QuantParams& p, cudaStream_t s) {
  quantize_kernel<F, R><<<grid, kQuantThreads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K) {
  (void)rows;
  (void)K;
  return sizeof(WorkspaceHeader) + sizeof(uint32_t) * kMaxPartials;
}

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                            int rule, float fp8_max, void* codes, void* scales,
                            float* global_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!x || !codes || !scales || !global_scale || !workspace)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: null pointer argument");
  if (rows < 1 || K < 64 || K % 64 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "nvfp4_quantize: need rows >= 1 and K a positive multiple of 64 (rows=%lld K=%lld)",
                     (long long)rows, (long long)K);
  if (ldx < K || ldx % 8 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: need ldx >= K and ldx %% 8 == 0");
  if (mode != NVFP4_MODE_SIX && mode != NVFP4_MODE_FOUR_OVER_SIX)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: unknown mode %d", mode);
  if (rule != NVFP4_RULE_MAX && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: unknown rule %d", rule);
  if (!(fp8_max == 448.0f || fp8_max == 256.0f))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: fp8_max must be 448 or 256");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3u))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: misaligned buffer");
  if (workspace_bytes < nvfp4_quantize_workspace_bytes(rows, K))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: workspace too small");
  const int64_t row_blocks = (rows + 127) / 128;
  const int64_t ntasks = row_blocks * 16 * (K / 64);
  if (ntasks > 0xFFFFFFFFll || rows * ldx > (1ll << 40))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize: tensor too large");
  int dev = 0, sms = 0;
  nvfp4_status st = check_device(&dev, &sms);
  if (st != NVFP4_OK) return st;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto* ws = static_cast<WorkspaceHeader*>(workspace);
  auto* partials = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + sizeof(WorkspaceHeader));

  int amax_grid;
  if (ldx == K) {
    const int64_t nvec = rows * K / 8;
    amax_grid = static_cast<int>(std::min<int64_t>((nvec + kAmaxThreads * 4 - 1) / (kAmaxThreads * 4),
                                                   static_cast<int64_t>(sms) * 4));
  } else {
    amax_grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(sms) * 4));
  }
  amax_grid = std::max(1, std::min(amax_grid, kMaxPartials));
  amax_kernel<<<amax_grid, kAmaxThreads, 0, s>>>(static_cast<const uint16_t*>(x), rows, K, ldx,
                                                  partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "amax_kernel launch");

  QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.rows = rows;
  p.K = K;
  p.ldx = ldx;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  p.global_scale = global_scale;
  p.partials = partials;
  p.ws = ws;
  p.nparts = amax_grid;
  p.f6 = fp8_max * 6.0f;
  p.ntasks = static_cast<uint32_t>(ntasks);
  p.kgroups = static_cast<uint32_t>(K / 64);
  const int64_t want = (ntasks + kQuantWarps - 1) / kQuantWarps;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * 8)));
  if (mode == NVFP4_MODE_SIX) e = launch_quantize<false, kRuleMax>(grid, p, s);
  else if (rule == NVFP4_RULE_MAX) e = launch_quantize<true, kRuleMax>(grid, p, s);
  else if (rule == NVFP4_RULE_MAE) e = launch_quantize<true, kRuleMae>(grid, p, s);
  else e = launch_quantize<true, kRuleMse>(grid, p, s);
  if (e != cudaSuccess) return cuda_status(e, "quantize_kernel launch");
  return NVFP4_OK;
}

}  // extern "C"

// ------------------------------------------------ allocation-free variant --
//
// nvfp4_quantize needs a caller-provided device workspace for the amax pass's
// per-CTA partial maxima and the status word.  Some callers cannot provide
// one: a custom-op or plugin hook running inside another inference runtime
// that owns every device allocation and hands the op only its inputs and
// outputs, or a service that fixes its device-memory footprint at start-up
// and must not allocate on the request path (an allocation there can block,
// fragment the pool, or fail under memory pressure in the middle of a
// request).  nvfp4_quantize_noalloc runs the same two kernels with that
// scratch in a static device array instead, so it allocates nothing.
//
// The array below is held by every GPU that loads this library, from module
// load until process exit.  Its size bounds the amax pass at kMaxPartials
// CTAs (the launch uses at most 4 per SM, 592 on a B200); a launch that would
// need more is rejected.  Nothing in it has to start at zero: each call's amax
// kernel writes every partial slot the following quantize kernel reads, and
// the quantize kernel writes the status word.  All calls on a device share it,
// so two calls that may overlap on the GPU (different streams without an
// ordering between them) race on it and must be serialized by the caller.

namespace nvfp4 {
namespace {

constexpr size_t kNoAllocScratchBytes = sizeof(WorkspaceHeader) + sizeof(uint32_t) * kMaxPartials;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void* g_noalloc_addr[kNoAllocMaxDevices];

// Device address of g_noalloc_scratch on the current device `dev`, looked up
// once per device (the first call on a device does this set-up).  In host
// code the array's name is only a host-side stand-in for the symbol, never a
// device address, so kernels must get this pointer instead.
nvfp4_status noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(NVFP4_ERR_UNSUPPORTED_DEVICE, "nvfp4_quantize_noalloc: device %d", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(noalloc scratch)");
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                               int mode, int rule, float fp8_max, void* codes,
                                               void* scales, float* global_scale, void* stream) {
  if (!x || !codes || !scales || !global_scale)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: null pointer argument");
  if (rows < 1 || K < 64 || K % 64 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "nvfp4_quantize_noalloc: need rows >= 1 and K a positive multiple of 64 (rows=%lld K=%lld)",
                     (long long)rows, (long long)K);
  if (ldx < K || ldx % 8 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: need ldx >= K and ldx %% 8 == 0");
  if (mode != NVFP4_MODE_SIX && mode != NVFP4_MODE_FOUR_OVER_SIX)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: unknown mode %d", mode);
  if (rule != NVFP4_RULE_MAX && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: unknown rule %d", rule);
  if (!(fp8_max == 448.0f || fp8_max == 256.0f))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: fp8_max must be 448 or 256");
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3u))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: misaligned buffer");
  const int64_t row_blocks = (rows + 127) / 128;
  const int64_t ntasks = row_blocks * 16 * (K / 64);
  if (ntasks > 0xFFFFFFFFll || rows * ldx > (1ll << 40))
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_quantize_noalloc: tensor too large");
  int dev = 0, sms = 0;
  nvfp4_status st = check_device(&dev, &sms);
  if (st != NVFP4_OK) return st;

  int amax_grid;
  if (ldx == K) {
    const int64_t nvec = rows * K / 8;
    amax_grid = static_cast<int>(std::min<int64_t>((nvec + kAmaxThreads * 4 - 1) / (kAmaxThreads * 4),
                                                   static_cast<int64_t>(sms) * 4));
  } else {
    amax_grid = static_cast<int>(std::min<int64_t>(rows, static_cast<int64_t>(sms) * 4));
  }
  amax_grid = std::max(1, amax_grid);
  if (amax_grid > kMaxPartials)
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "nvfp4_quantize_noalloc: the amax pass needs %d partial slots but the static "
                     "scratch holds %d (%zu bytes)", amax_grid, kMaxPartials, kNoAllocScratchBytes);

  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != NVFP4_OK) return st;
  auto* ws = static_cast<WorkspaceHeader*>(scratch);
  auto* partials = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + sizeof(WorkspaceHeader));

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  amax_kernel<<<amax_grid, kAmaxThreads, 0, s>>>(static_cast<const uint16_t*>(x), rows, K, ldx,
                                                  partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "amax_kernel launch");

  QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.rows = rows;
  p.K = K;
  p.ldx = ldx;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  p.global_scale = global_scale;
  p.partials = partials;
  p.ws = ws;
  p.nparts = amax_grid;
  p.f6 = fp8_max * 6.0f;
  p.ntasks = static_cast<uint32_t>(ntasks);
  p.kgroups = static_cast<uint32_t>(K / 64);
  const int64_t want = (ntasks + kQuantWarps - 1) / kQuantWarps;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * 8)));
  if (mode == NVFP4_MODE_SIX) e = launch_quantize<false, kRuleMax>(grid, p, s);
  else if (rule == NVFP4_RULE_MAX) e = launch_quantize<true, kRuleMax>(grid, p, s);
  else if (rule == NVFP4_RULE_MAE) e = launch_quantize<true, kRuleMae>(grid, p, s);
  else e = launch_quantize<true, kRuleMse>(grid, p, s);
  if (e != cudaSuccess) return cuda_status(e, "quantize_kernel launch");
  return NVFP4_OK;
}
