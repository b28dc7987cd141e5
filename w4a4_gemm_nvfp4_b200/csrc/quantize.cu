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
// The 16 values of a block are held as binary32 pairs (x_j, x_{j+8}) and the
// per-element arithmetic uses packed f32x2 instructions (each lane an IEEE RNE
// operation, like the scalar one); with that pairing the contiguous pairwise
// error sum is three packed additions and one scalar one.
//
// Two kernels per call:
//   amax_kernel      one HBM read of x; each CTA writes the max |bf16| bit
//                    pattern it saw to a partials array in the workspace.
//   quantize_kernel  reduces the partials (a few KB, L2-resident) to alpha in
//                    every CTA, then makes one HBM pass over x: each lane owns
//                    one whole 16-element block (one 32-byte load), so the
//                    block max and both candidates' errors stay in registers
//                    with no shuffles.  A warp task is a pair of chunks of 32
//                    consecutive blocks (2 x 1 KB of x) of one row, and the
//                    warps of the grid take the tasks in a sweep, so x is read
//                    front to back; every lane writes its 8 code bytes and its
//                    scale byte at that block's place in the swizzled scale
//                    layout.
// The other entry points reuse the block step: quantize_t_kernel (blocks down
// the columns of x, through shared-memory tiles), quantize_arc_kernel
// (reordered channels plus appended residual or duplicated ones, with an
// optional RMSNorm of the activations) and its RMS pass (rms_amax_reg_kernel
// with the row in registers up to K = 8192, rms_amax_kernel above).
#include <cuda_fp16.h>

#include <algorithm>

#include "block_step.cuh"
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kAmaxThreads = 512;
constexpr int kMaxPartials = 4096;
constexpr size_t align16(size_t n) { return (n + 15) & ~static_cast<size_t>(15); }
constexpr int kArcMaxRows = 4;              // rows per step of the augmented quantizer, at most
constexpr int kArcPrimThreads = 256;        // its threads for the primary blocks, at most
constexpr int kArcMaxThreads = 640;         // its block size, at most
constexpr int kArcMaxBufs = 3;              // its row buffers: 3, or 2 for the widest rows
constexpr int64_t kArcSmemStep = 73728;     // shared memory it aims at: three CTAs per SM up to 5K channels
constexpr int64_t kArcMaxK = 16384;         // channels of x it takes, at most
// its dynamic shared memory opt-in: 2 bytes x K x (1 + buffers x rows per step), the offsets
// ahead of the row buffers, is at most 2 x 16384 x 3 (two buffers of one row)
constexpr int64_t kArcSmemBudget = 2 * 16384 * 4;
constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// ------------------------------------------------------------- amax pass --
// Magnitudes compare like their bit patterns once the sign is cleared, and
// every NaN pattern (> 0x7F80) compares above Inf (0x7F80) above any finite
// value, so one unsigned max gives both amax and the non-finite flag.  Each
// thread keeps eight 16-byte loads in flight; two 512-thread CTAs per SM.
// The pass walks x from its end, so that its last reads -- the front of x,
// where the quantize kernel starts -- are the ones still in L2 (measured: 4/6
// amax + quantize 2 us faster on a 32768 x 5120 x).
__global__ void __launch_bounds__(kAmaxThreads, 2)
    amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                uint32_t* __restrict__ partials) {
  pdl_launch_dependents();  // the quantize kernel may be scheduled now; it waits for this grid's end
  uint32_t m = 0;
  if (ldx == K) {
    const uint4* v = reinterpret_cast<const uint4*>(x);
    const int64_t n = rows * K / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + 7 * stride < n; i += 8 * stride) {
      uint4 a[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) a[u] = ld_stream(v + (n - 1 - (i + u * stride)));
#pragma unroll
      for (int u = 0; u < 8; ++u) m = absmax4(a[u], m);
    }
    for (; i < n; i += stride) m = absmax4(ld_stream(v + (n - 1 - i)), m);
  } else {
    const int64_t k8 = K / 8;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
      const uint4* v = reinterpret_cast<const uint4*>(x + (rows - 1 - r) * ldx);
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

struct QuantParams {
  const uint16_t* x;
  int64_t rows, K, ldx;
  uint8_t* codes;
  uint8_t* scales;
  float* global_scale;
  const uint32_t* partials;   // amax partials (dynamic alpha) ...
  const float* alpha_in;      // ... or a caller-supplied alpha (static), else null
  WorkspaceHeader* ws;
  int nparts;
  float f6;            // fp8_max * 6
  uint32_t ntasks;     // row-wise kernel: 512-element chunks over the rows padded to 128
  uint32_t chunks;     // row-wise kernel: chunks per row, ceil(K / 512)
  uint32_t kgroups;    // K / 64
  // augmented (ARCQuant) quantization only
  const int32_t* perm = nullptr;  // channel order, K entries
  int64_t S = 0;                  // augmented channels
  int augment = 0;                // 0: residual of the first S reordered channels, 1: their copy
  int arc_rows = 1;               // rows per step of the augmented quantizer
  int arc_prim_threads = 128;     // its threads for the primary blocks; the rest take the appended ones
  int arc_bufs = 3;               // its row buffers
  // RMSNorm ahead of the augmented quantizer only
  const uint16_t* gamma = nullptr;  // bf16 gains, K entries
  const float* rinv = nullptr;      // 1 / rms of each row, written by the RMS pass
  const uint16_t* gperm = nullptr;  // the gains in channel order (gamma[perm[i]]), written by the RMS pass
};

// Start of every quantize kernel: alpha (a caller-supplied static scale, or
// the tensor amax reduced from the partials of the amax pass -- every CTA
// reduces the same partials), the per-call constants of the block step and
// the (d, r) table of every E4M3 scale code.  The block size is a multiple of
// 32 and at least 128 (the table has one entry per thread of the first 128).  Returns false when the kernel
// must stop (non-finite tensor, invalid static alpha); that is uniform over
// the grid.
__device__ __forceinline__ bool quant_prologue(const QuantParams& p, BlockConsts& k, ScaleEntry* s_dr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // launched as a programmatic dependent of the amax pass (dynamic alpha):
  // let the next kernel be scheduled, then wait for the amax pass to finish
  // before reading its partials, and before any other access to memory
  pdl_launch_dependents();
  pdl_wait();
  float alpha;
  if (p.alpha_in) {
    alpha = __ldg(p.alpha_in);
    if (!(alpha > 0.0f) || isinf(alpha)) {  // not a positive finite number
      if (blockIdx.x == 0 && threadIdx.x == 0) p.ws->status = NVFP4_ERR_INVALID_ARG;
      return false;
    }
    // the status word was cleared to NVFP4_OK before the launch; CTAs only
    // ever raise it (to NVFP4_ERR_NONFINITE), so their order does not matter
  } else {
    __shared__ uint32_t s_red[32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < p.nparts; i += blockDim.x) m = max(m, p.partials[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    uint32_t amax_bits = 0;
#pragma unroll
    for (int w = 0; w < 32; ++w)
      if (w < static_cast<int>(blockDim.x >> 5)) amax_bits = max(amax_bits, s_red[w]);
    const bool nonfinite = amax_bits >= 0x7F80u;
    alpha = amax_bits == 0 ? 1.0f : __fdiv_rn(__uint_as_float(amax_bits << 16), p.f6);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.ws->status = nonfinite ? NVFP4_ERR_NONFINITE : NVFP4_OK;
      p.ws->detail = amax_bits;
      *p.global_scale = nonfinite ? __uint_as_float(0x7FC00000u) : alpha;
    }
    if (nonfinite) return false;
  }
  make_block_consts(alpha, k);
  fill_scale_table(alpha, s_dr, threadIdx.x);  // constants of every E4M3 scale code
  __syncthreads();
  return true;
}

// Warp tasks of the row-wise kernel: pairs of chunks of 32 consecutive
// 16-element blocks (2 x 512 elements, 2 KB of x) of one row; lane i takes
// block i of each chunk, first chunk 2j, then chunk 2j+1 (absent when a row
// has an odd number of chunks; the last chunk of a row is partial when
// K % 512 != 0).  Tasks are numbered row-major over the rows padded to a
// multiple of 128, and the W warps of the grid take them in a sweep (warp g:
// tasks g, g + W, g + 2W, ...), so at any moment they work on neighbouring
// chunks and the grid reads x front to back as one stream (measured 93 % of
// the copy bandwidth for the bare load/store loop, against 83-86 % when each
// warp or CTA walks a region of its own).  A step of W tasks is a fixed number
// of rows and chunk pairs, so the row and the lane's pointers into x and the
// codes advance by precomputed increments (one of two, depending on whether
// the pair index wrapped); the second chunk of a task is at fixed offsets from
// the first, so the bookkeeping of a task is paid once per two blocks.  Each
// lane loads its next block (the task's second one, or the next task's first)
// while it quantizes the current one.  Rows past `rows` only write their
// (zero) scale bytes.
// A block's 32 bytes: one 256-bit load when V8 (p 32-byte aligned; the
// sector then crosses from L2 once, where two non-allocating 128-bit loads
// each fetch it), else two 128-bit loads.
template <bool V8>
__device__ __forceinline__ void ld_block2(const uint16_t* p, uint4& lo, uint4& hi) {
  if constexpr (V8) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
                 : "l"(p));
  } else {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    lo = ld_stream(q);
    hi = ld_stream(q + 1);
  }
}

__device__ __forceinline__ int64_t scale_row_offset(uint32_t row, uint32_t kgroups) {
  return static_cast<int64_t>(row >> 7) * kgroups * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4;
}

template <bool FOUR_OVER_SIX, int RULE, bool V8>
// Scale-6: four CTAs per SM (64 registers), measured faster than three, five
// or six.  Four-Over-Six: three CTAs per SM (up to 85 registers), which keeps
// its two candidates' state out of local memory; measured 2-3 % faster than
// four with spills.
__global__ void __launch_bounds__(kQuantThreads, FOUR_OVER_SIX ? 3 : 4)
    quantize_kernel(const QuantParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  BlockConsts k;
  __shared__ ScaleEntry s_dr[128];
  if (!quant_prologue(p, k, s_dr)) return;

  const uint32_t nwarps = gridDim.x * kQuantWarps;
  uint32_t t = blockIdx.x * kQuantWarps + warp;  // < 2^31: t + nwarps does not wrap
  if (t >= p.ntasks) return;
  const uint32_t cpr = p.chunks;                       // chunks per row
  const uint32_t ppr = (cpr + 1) / 2;                  // chunk pairs (tasks) per row
  const uint32_t kbs = static_cast<uint32_t>(p.K / 16);
  // whether this lane has a block in chunk c of a row
  const bool lane_in_last = static_cast<uint32_t>(lane) < kbs - (cpr - 1) * 32;
  auto has_block = [&](uint32_t c) { return c + 1 < cpr || (c + 1 == cpr && lane_in_last); };
  const uint32_t rows = static_cast<uint32_t>(p.rows);  // < 2^31 (ntasks < 2^31)
  // one sweep step = drow rows + dpair chunk pairs; the pointer increments for
  // a step without and with a pair-index wrap (the next row's first pairs)
  const uint32_t drow = nwarps / ppr, dpair = nwarps - drow * ppr;
  const int64_t half_k = p.K / 2;
  const int64_t dx = static_cast<int64_t>(drow) * p.ldx + dpair * 1024;
  const int64_t dx_wrap = dx + p.ldx - static_cast<int64_t>(ppr) * 1024;
  const int64_t dc = static_cast<int64_t>(drow) * half_k + dpair * 512;
  const int64_t dc_wrap = dc + half_k - static_cast<int64_t>(ppr) * 512;
  uint32_t row = t / ppr, pair = t - row * ppr;
  const uint16_t* xp = p.x + static_cast<int64_t>(row) * p.ldx + pair * 1024 + lane * 16;
  uint8_t* cp = p.codes + static_cast<int64_t>(row) * half_k + pair * 512 + lane * 8;
  uint8_t* const sp = p.scales + static_cast<uint32_t>(lane >> 2) * 512 + (lane & 3);

  // quantize one block (loaded in lo/hi) of row `r` at codes `c` and scale `s`
  auto block = [&](const uint4& lo, const uint4& hi, uint32_t r, uint8_t* c, uint8_t* s) {
    uint32_t scale = 0;
    if (r < rows) {
      uint2 codes;
      const uint32_t bmax = quantize_block<FOUR_OVER_SIX, RULE>(lo, hi, k, s_dr, codes, scale);
      if (p.alpha_in && bmax >= 0x7F80u) {
        // Inf/NaN in this block (a static alpha skips the tensor check):
        // the block is written as zeros and the call reports it
        codes = make_uint2(0u, 0u);
        scale = 0u;
        p.ws->status = NVFP4_ERR_NONFINITE;
      }
      *reinterpret_cast<uint2*>(c) = codes;
    }
    *s = static_cast<uint8_t>(scale);
  };

  // (a block register pair is only used when its block is quantized, and such
  // a block was always loaded; they are zeroed once so that no copy of them
  // is ever of an indeterminate value)
  uint4 lo = make_uint4(0, 0, 0, 0), hi = lo, nlo = lo, nhi = lo;
  if (row < rows && has_block(2 * pair)) ld_block2<V8>(xp, lo, hi);
  for (;;) {
    const uint32_t cur_row = row, c0 = 2 * pair;
    const uint16_t* const cur_xp = xp;
    uint8_t* const cur_cp = cp;
    uint8_t* const cur_sp = sp + scale_row_offset(cur_row, p.kgroups) + c0 * 4096;
    // first chunk of the pair, while the second one loads
    const bool second = has_block(c0 + 1);
    if (cur_row < rows && second) ld_block2<V8>(cur_xp + 512, nlo, nhi);
    if (has_block(c0)) block(lo, hi, cur_row, cur_cp, cur_sp);
    // advance to the next task
    t += nwarps;
    row += drow;
    pair += dpair;
    const bool wrap = pair >= ppr;
    if (wrap) {
      pair -= ppr;
      ++row;
    }
    xp += wrap ? dx_wrap : dx;
    cp += wrap ? dc_wrap : dc;
    const bool more = t < p.ntasks;
    // second chunk, while the next task's first chunk loads
    if (more && row < rows && has_block(2 * pair)) ld_block2<V8>(xp, lo, hi);
    if (second) block(nlo, nhi, cur_row, cur_cp + 256, cur_sp + 4096);
    if (!more) break;
  }
}

// Quantization of x^T: the NVFP4 operand of the [K, rows] matrix x^T, i.e.
// 16-element blocks along rows (a column of x), as the weight-gradient and
// input-gradient GEMMs of training need it.  A CTA walks 128-row x 64-column
// tiles of x (grid-stride).  Each tile is copied into shared memory with
// 16-byte asynchronous copies (cp.async; chunks outside x are zero-filled),
// chunk index XOR-swizzled by the 16-row group so the column reads below hit
// 32 distinct banks; two tile buffers are used in turn, so the next tile's
// copies are in flight while the current one is quantized.  Thread t
// quantizes the two columns 2(t>>3), 2(t>>3)+1 over rows 16(t&7) ..
// 16(t&7)+15 with the same block step as the row-wise kernel.
// Output row kk of x^T, block mb: codes at kk*(rows/2) + 8*mb, scale in the
// swizzled layout of a [K, rows] operand; rows kk in [K, ceil(K/128)*128)
// get zero scales.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  // src-size 0 copies nothing and zero-fills the 16 bytes
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
// Plain arrive (count 1) on a shared::cta mbarrier.
__device__ __forceinline__ void mbar_arrive_local(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on the mbarrier `bar`.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// 16-bit shared-memory load at a 32-bit shared address (zero-extended);
// volatile, so it is not moved across the barriers that publish the rows
__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <bool FOUR_OVER_SIX, int RULE>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_t_kernel(const QuantParams p) {
  BlockConsts k;
  __shared__ ScaleEntry s_dr[128];
  __shared__ __align__(16) uint32_t tile[2][128 * 32];  // two buffers of 128 rows x 128 bytes
  if (!quant_prologue(p, k, s_dr)) return;

  const int64_t M = p.rows, K = p.K;
  const int64_t k_pad = (K + 127) / 128 * 128;
  const uint32_t tiles_m = static_cast<uint32_t>((M + 127) / 128);
  const uint32_t tiles_k = static_cast<uint32_t>(k_pad / 64);
  const uint32_t ntiles = tiles_m * tiles_k;
  const int cp = threadIdx.x >> 3, mb = threadIdx.x & 7;
  const int64_t half_m = M / 2;
  const int64_t kgroups_t = M / 64;  // K groups of the transposed operand
  // issue the copies of tile `t` into buffer `b` (4 chunks of 16 bytes per thread)
  auto load_tile = [&](uint32_t t, int b) {
    const int64_t m0 = static_cast<int64_t>(t % tiles_m) * 128;
    const int64_t k0 = static_cast<int64_t>(t / tiles_m) * 64;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = threadIdx.x + i * kQuantThreads;
      const int r = q >> 3, ch = q & 7;
      const bool valid = m0 + r < M && k0 + ch * 8 < K;
      const uint16_t* src = valid ? p.x + (m0 + r) * p.ldx + k0 + ch * 8 : p.x;
      cp_async16(smem_u32(&tile[b][r * 32 + ((ch ^ ((r >> 4) & 7)) << 2)]), src, valid);
    }
    cp_async_commit();
  };
  uint32_t t = blockIdx.x;
  if (t >= ntiles) return;
  load_tile(t, 0);
  for (int b = 0;; b ^= 1) {
    const uint32_t next = t + gridDim.x;
    if (next < ntiles) {
      load_tile(next, b ^ 1);
      cp_async_wait<1>();  // this tile's copies have landed (the next tile's may still fly)
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int64_t m0 = static_cast<int64_t>(t % tiles_m) * 128;
    const int64_t k0 = static_cast<int64_t>(t / tiles_m) * 64;
    // ---- two column blocks per thread ----
    const int64_t mb_g = m0 / 16 + mb;
    if (mb_g * 16 < M) {
      const uint32_t* tl = tile[b];
      uint32_t wl[8], wh[8];  // column 2cp / 2cp+1 as bf16 pairs (element 2i in the low half)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int r0 = mb * 16 + 2 * i;
        const uint32_t a = tl[r0 * 32 + (((cp >> 2) ^ mb) << 2) + (cp & 3)];
        const uint32_t c = tl[(r0 + 1) * 32 + (((cp >> 2) ^ mb) << 2) + (cp & 3)];
        wl[i] = __byte_perm(a, c, 0x5410);
        wh[i] = __byte_perm(a, c, 0x7632);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t kk = k0 + 2 * cp + h;
        if (kk >= k_pad) continue;
        uint32_t scale = 0;
        if (kk < K) {
          const uint32_t* w = h ? wh : wl;
          const uint4 lo = make_uint4(w[0], w[1], w[2], w[3]), hi = make_uint4(w[4], w[5], w[6], w[7]);
          uint2 codes;
          const uint32_t bmax = quantize_block<FOUR_OVER_SIX, RULE>(lo, hi, k, s_dr, codes, scale);
          if (p.alpha_in && bmax >= 0x7F80u) {
            codes = make_uint2(0u, 0u);
            scale = 0u;
            p.ws->status = NVFP4_ERR_NONFINITE;
          }
          *reinterpret_cast<uint2*>(p.codes + kk * half_m + mb_g * 8) = codes;
        }
        const int64_t atom = (kk >> 7) * kgroups_t + (mb_g >> 2);
        p.scales[atom * 512 + (kk & 31) * 16 + ((kk >> 5) & 3) * 4 + (mb_g & 3)] =
            static_cast<uint8_t>(scale);
      }
    }
    if (next >= ntiles) break;
    __syncthreads();  // every thread has read this buffer before it is refilled
    t = next;
  }
}

// ------------------------------------------------------------- RMS pass --
// RMSNorm ahead of the augmented quantizer (ARCQuant page, 방법론, 커널
// 구현: the fused kernel normalizes the activations before reordering and
// quantizing them; the page gives no formula, so this is the standard RMSNorm,
// each step one binary32 operation):
//   r = 1 / sqrt(sum_k x_k^2 / K + eps),  y_k = bf16((x_k * r) * gamma_k)
// with the sum of squares taken as the contiguous pairwise tree over the row
// (zero-padded to a power of two P).  One warp per row, no block barrier: in
// round q the warp reads 1024 consecutive elements, lane l the four 16-byte
// groups 128q + 4l .. 128q + 4l + 3 (64 contiguous bytes; the warp's four
// loads cover 2 KB), sums its 32 squares as a pairwise tree, and an xor
// butterfly over the lanes combines the lanes' adjacent subtrees (1, then 2,
// 4, ... lanes: the same tree, addition being commutative).  The rounds'
// sums, all lanes holding them, merge like a binary counter (each completed
// subtree added to the equal-size one on its left); the zero padding past the
// last round is not computed.  Every lane ends with the row's sum and computes
// r.  The pass writes r for every row, the gains in channel order and, like
// the amax pass, each CTA's max |bf16(y)| as a bit pattern (from the bound of
// rms_row_max_bits, without computing y where the bound decides).
constexpr int kRmsThreads = 256;
constexpr int kRmsRegThreads = 128;

// two binary32 values -> a bf16 pair (lo in the low half), nearest, ties to even
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t w;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w) : "f"(hi), "f"(lo));
  return w;
}

// the squares of a bf16 pair, each rounded once to binary32 (the mixed-precision
// fma computes x * x + (-0) exactly and rounds it: the binary32 product)
__device__ __forceinline__ void sq_pair(uint32_t w, float& lo, float& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "fma.rn.f32.bf16 %0, l, l, 0f80000000;\n\t"
      "fma.rn.f32.bf16 %1, h, h, 0f80000000;\n\t}"
      : "=f"(lo), "=f"(hi)
      : "r"(w));
}

// the squares of the 8 bf16 values of one 16-byte group, summed as a pairwise tree
__device__ __forceinline__ float sq_tree8(const uint4 v) {
  float a[8];
  sq_pair(v.x, a[0], a[1]);
  sq_pair(v.y, a[2], a[3]);
  sq_pair(v.z, a[4], a[5]);
  sq_pair(v.w, a[6], a[7]);
  // first level in packed pairs: (a0 + a1, a2 + a3) and (a4 + a5, a6 + a7)
  const f2 b01 = add2(make_f2(a[0], a[2]), make_f2(a[1], a[3]));
  const f2 b23 = add2(make_f2(a[4], a[6]), make_f2(a[5], a[7]));
  return __fadd_rn(__fadd_rn(b01.a(), b01.b()), __fadd_rn(b23.a(), b23.b()));
}

// max(m, |(x * r) * gamma|) over one 16-byte group of x and its gains, in
// binary32 before the bf16 rounding: rounding to nearest is monotone and odd,
// so the largest |bf16(y)| is bf16 of the largest |y| and the pass rounds once
__device__ __forceinline__ float rms_group_max(const uint4 xv, const uint4 gv, f2 rr, float m) {
  const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const f2 xf = make_f2(__uint_as_float(xs[i] << 16), __uint_as_float(xs[i] & 0xFFFF0000u));
    const f2 gf = make_f2(__uint_as_float(gs[i] << 16), __uint_as_float(gs[i] & 0xFFFF0000u));
    const f2 y = mul2(mul2(xf, rr), gf);
    m = max3_nan(m, fabsf(y.a()), fabsf(y.b()));
  }
  return m;
}

// one round: the sum of this lane's four groups (32 contiguous elements; s_u
// the pairwise sum of group u) as a pairwise tree, combined over the warp by the xor butterfly (a 1024-element
// subtree; zero groups past the row add exact zeros)
__device__ __forceinline__ float rms_round(float s0, float s1, float s2, float s3) {
  float v = __fadd_rn(__fadd_rn(s0, s1), __fadd_rn(s2, s3));
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// round q's subtree into the binary counter: each completed subtree is added
// to the equal-size one on its left (q < 16)
__device__ __forceinline__ void rms_push(float (&stk)[5], int q, float v) {
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    if (!((q >> lvl) & 1)) {
      stk[lvl] = v;
      break;
    }
    v = __fadd_rn(stk[lvl], v);
  }
}

// the row's sum after `used` rounds: the counter holds one complete subtree
// per set bit of `used`, the lowest bit's the rightmost; the zero padding up
// to the next power of two leaves each the left operand of all to its right
__device__ __forceinline__ float rms_close(const float (&stk)[5], int used) {
  float v = 0.0f;
  bool have = false;
#pragma unroll
  for (int lvl = 0; lvl < 5; ++lvl) {
    if ((used >> lvl) & 1) {
      v = have ? __fadd_rn(stk[lvl], v) : stk[lvl];
      have = true;
    }
  }
  return v;
}

// r = 1 / sqrt(sum / K + eps), each step one rounding
__device__ __forceinline__ float rms_rinv(float sum, int64_t K, float eps) {
  return __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(sum, static_cast<float>(K)), eps)));
}

// the CTA's max |bf16(y)| from each lane's (a bf16 bit pattern without its
// sign; a NaN is 0x7FFF and compares above every number) into partials[blockIdx.x]
template <int THREADS>
__device__ __forceinline__ void rms_write_partial(uint32_t mb, uint32_t* partials) {
  const int lane = static_cast<int>(threadIdx.x & 31), warp = static_cast<int>(threadIdx.x >> 5);
#pragma unroll
  for (int o = 16; o; o >>= 1) mb = max(mb, __shfl_xor_sync(0xffffffffu, mb, o));
  __shared__ uint32_t s_max[THREADS / 32];
  if (lane == 0) s_max[warp] = mb;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t mm = 0;
    for (int w = 0; w < THREADS / 32; ++w) mm = max(mm, s_max[w]);
    partials[blockIdx.x] = mm;
  }
}

// gperm[i] = gamma[perm[i]] over the grid's threads, for the augmented
// quantizer's RMSNorm (an out-of-range channel reads channel 0, as there)
__device__ __forceinline__ void rms_permute_gains(const uint16_t* gamma, const int32_t* perm, int64_t K,
                                                  uint16_t* gperm) {
  const int64_t n = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < K; i += n) {
    const int32_t c = perm[i];
    gperm[i] = gamma[c >= 0 && c < K ? c : 0];
  }
}

// max(m, |x * gamma|) over one 16-byte group: each product of two bf16 values
// by one mixed-precision fma (exact: at most 16 significant bits, unless it
// falls below the binary32 normal range)
__device__ __forceinline__ float prod_group_max(const uint4 xv, const uint4 gv, float m) {
  const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, gs[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float t0, t1;
    asm("{\n\t.reg .b16 xl, xh, gl, gh;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "mov.b32 {gl, gh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, xl, gl, 0f80000000;\n\t"
        "fma.rn.f32.bf16 %1, xh, gh, 0f80000000;\n\t}"
        : "=f"(t0), "=f"(t1)
        : "r"(xs[i]), "r"(gs[i]));
    m = max3_nan(m, fabsf(t0), fabsf(t1));
  }
  return m;
}

__device__ __forceinline__ float warp_max_nan(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = max3_nan(v, __shfl_xor_sync(0xffffffffu, v, o), v);
  return v;
}

// Two adjacent 16-byte groups (32 bytes at p): one 256-bit load when V8 (p
// 32-byte aligned), else two 128-bit loads.  The 256-bit form halves the L1
// sector lookups of the lane pattern below (lanes 64 bytes apart).  VOL keeps
// a load in the loop for data that is the same every row (the gains), which
// would otherwise be hoisted into registers the row needs.
template <bool V8, bool VOL>
__device__ __forceinline__ void ld_group_pair(const uint16_t* p, uint4& a, uint4& b) {
  if constexpr (V8 && VOL) {
    asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
  } else if constexpr (V8) {
    asm("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
        : "l"(p));
  } else {
    a = reinterpret_cast<const uint4*>(p)[0];
    b = reinterpret_cast<const uint4*>(p)[1];
  }
}

// Whether max |gamma| <= 2^20 (NaN counts as not), over the warp: the bound
// on a row's max |y| below is only used then.
__device__ __forceinline__ bool rms_gains_small(const uint16_t* gamma, int64_t K, int lane) {
  uint32_t gb = 0;  // max |gamma| as bf16 bits (a NaN compares above every number)
  for (int64_t k = 8 * lane; k < K; k += 256) gb = absmax4(*reinterpret_cast<const uint4*>(gamma + k), gb);
#pragma unroll
  for (int o = 16; o; o >>= 1) gb = max(gb, __shfl_xor_sync(0xffffffffu, gb, o));
  return max(gb & 0xFFFFu, gb >> 16) <= 0x4980u;  // 2^20
}

// max |bf16(y)| of row xr as a bf16 bit pattern, y = (x * r) * gamma with two
// roundings, from P = max |x * gamma| over the row (exact) and r.  With every
// y in the normal range, each |y| is within a factor (1 +- 2^-24)^2 of
// |x * gamma| * r, so max |y| lies in [lo, hi] = [P r (1 - 2^-20), P r (1 + 2^-20)]
// (rounded outward; the slack also covers what underflow can add while
// P r >= 2^-90 and max |gamma| <= 2^20).  Rounding to bf16 is monotone and
// odd: when lo and hi round to the same bf16 value, that is the answer;
// otherwise (about one row in two thousand), or outside those ranges, the row
// is read again and its y computed one by one.  Warp-uniform.
__device__ __forceinline__ uint32_t rms_row_max_bits(float P, float rr, bool gains_small, const uint16_t* xr,
                                                     const uint16_t* gamma, int64_t K, int lane) {
  const float plo = __fmul_rd(P, rr), phi = __fmul_ru(P, rr);
  const uint32_t blo = bf16x2_rn(__fmul_rd(plo, 1.0f - 0x1p-20f), 0.0f) & 0x7FFFu;
  const uint32_t bhi = bf16x2_rn(__fmul_ru(phi, 1.0f + 0x1p-20f), 0.0f) & 0x7FFFu;
  if (gains_small && plo >= 0x1p-90f && P <= 0x1.fffffep127f && blo == bhi) return blo;
  const f2 rrr = make_f2(rr, rr);
  float m = 0.0f;
#pragma unroll 1
  for (int64_t k = 8 * lane; k < K; k += 256)
    m = rms_group_max(*reinterpret_cast<const uint4*>(xr + k), *reinterpret_cast<const uint4*>(gamma + k), rrr, m);
  return bf16x2_rn(m, 0.0f) & 0x7FFFu;  // this lane's part; the partial takes the max over lanes
}

// The RMS pass with the row held in registers (K <= 1024 * NR): a warp issues
// every load of its row before any arithmetic, so the whole row is in flight
// at once, and the sum of squares and P come from the same registers.
template <int NR, bool V8>
__global__ void __launch_bounds__(kRmsRegThreads, NR <= 2 ? 8 : NR <= 3 ? 5 : NR <= 6 ? 4 : 3)
    rms_amax_reg_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                        const uint16_t* __restrict__ gamma, float eps, const int32_t* __restrict__ perm,
                        float* __restrict__ rinv, uint16_t* __restrict__ gperm, uint32_t* __restrict__ partials) {
  pdl_launch_dependents();
  rms_permute_gains(gamma, perm, K, gperm);
  constexpr int kWarps = kRmsRegThreads / 32;
  const int lane = static_cast<int>(threadIdx.x & 31), warp = static_cast<int>(threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
  const bool gains_small = rms_gains_small(gamma, K, lane);
  uint32_t mb = 0;  // this lane's max |bf16(y)| as a bf16 bit pattern
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps + warp; r < rows; r += nwarps) {
    const uint16_t* xr = x + r * ldx;
    // (K % 64 == 0: a pair of groups is inside the row or past it)
    uint4 d[NR][4];
#pragma unroll
    for (int q = 0; q < NR; ++q) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k = 1024 * q + 32 * lane + 16 * h;
        if (k < K) {
          ld_group_pair<V8, false>(xr + k, d[q][2 * h], d[q][2 * h + 1]);
        } else {
          d[q][2 * h] = make_uint4(0u, 0u, 0u, 0u);
          d[q][2 * h + 1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    // the sum of squares and, from the same registers, P = max |x * gamma|
    float stk[5];
    float P = 0.0f;
#pragma unroll
    for (int q = 0; q < NR; ++q) {
      float g[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k = 1024 * q + 32 * lane + 16 * h;
        g[2 * h] = sq_tree8(d[q][2 * h]);
        g[2 * h + 1] = sq_tree8(d[q][2 * h + 1]);
        if (k < K) {
          uint4 ga, gb2;
          ld_group_pair<V8, true>(gamma + k, ga, gb2);
          P = prod_group_max(d[q][2 * h + 1], gb2, prod_group_max(d[q][2 * h], ga, P));
        }
      }
      rms_push(stk, q, rms_round(g[0], g[1], g[2], g[3]));
    }
    const float rr = rms_rinv(rms_close(stk, NR), K, eps);
    if (lane == 0) rinv[r] = rr;
    mb = max(mb, rms_row_max_bits(warp_max_nan(P), rr, gains_small, xr, gamma, K, lane));
  }
  rms_write_partial<kRmsRegThreads>(mb, partials);
}

// The RMS pass for any K <= 16384, round by round: each round's loads, its
// subtree of the sum and its part of P, then the next round.
template <bool V8>
__global__ void __launch_bounds__(kRmsThreads)
    rms_amax_kernel(const uint16_t* __restrict__ x, int64_t rows, int64_t K, int64_t ldx,
                    const uint16_t* __restrict__ gamma, float eps, const int32_t* __restrict__ perm,
                    float* __restrict__ rinv, uint16_t* __restrict__ gperm, uint32_t* __restrict__ partials) {
  pdl_launch_dependents();  // the quantize kernel may be scheduled now; it waits for this grid's end
  rms_permute_gains(gamma, perm, K, gperm);
  // rounds that hold elements; the zero-padded rest of the tree up to the next
  // power of two adds exact zeros and is not computed
  const int used = static_cast<int>((K + 1023) / 1024);  // 1 .. 16 (K <= 16384)
  const int lane = static_cast<int>(threadIdx.x & 31), warp = static_cast<int>(threadIdx.x >> 5);
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kRmsThreads / 32);
  const bool gains_small = rms_gains_small(gamma, K, lane);
  uint32_t mb = 0;
  for (int64_t r = static_cast<int64_t>(blockIdx.x) * (kRmsThreads / 32) + warp; r < rows; r += nwarps) {
    const uint16_t* xr = x + r * ldx;
    float stk[5];
    float P = 0.0f;
#pragma unroll 2  // two rounds' loads in flight (83.6 against 87.6 us on 8192 x 16384)
    for (int q = 0; q < used; ++q) {
      // this lane's two pairs of groups (K % 64 == 0: a pair is inside the row or past it)
      float g[4];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int64_t k = 1024 * static_cast<int64_t>(q) + 32 * lane + 16 * h;
        if (k < K) {
          uint4 a, b, ga, gb;
          ld_group_pair<V8, false>(xr + k, a, b);
          ld_group_pair<V8, true>(gamma + k, ga, gb);
          g[2 * h] = sq_tree8(a);
          g[2 * h + 1] = sq_tree8(b);
          P = prod_group_max(b, gb, prod_group_max(a, ga, P));
        } else {
          g[2 * h] = 0.0f;
          g[2 * h + 1] = 0.0f;
        }
      }
      rms_push(stk, q, rms_round(g[0], g[1], g[2], g[3]));
    }
    const float rr = rms_rinv(rms_close(stk, used), K, eps);
    if (lane == 0) rinv[r] = rr;
    mb = max(mb, rms_row_max_bits(warp_max_nan(P), rr, gains_small, xr, gamma, K, lane));
  }
  rms_write_partial<kRmsThreads>(mb, partials);
}

// A block's 16 gains in channel order (two 16-byte loads of gamma[perm[.]])
// as binary32 pairs, gv[i] = (gain 2i, gain 2i + 1).
__device__ __forceinline__ void rms_gains(const uint16_t* gperm, int j, f2 gv[8]) {
  const uint4 g0 = __ldg(reinterpret_cast<const uint4*>(gperm + 16 * j));
  const uint4 g1 = __ldg(reinterpret_cast<const uint4*>(gperm + 16 * j) + 1);
  const uint32_t gw[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) gv[i] = make_f2(__uint_as_float(gw[i] << 16), __uint_as_float(gw[i] & 0xFFFF0000u));
}

// The RMSNorm of a gathered block: x (8 bf16 pairs, element 2i low) becomes
// bf16((x * r) * gamma) with the block's gains gv (from rms_gains), as the RMS
// pass computes it; packed products are one RNE binary32 product per lane.
__device__ __forceinline__ void rms_normalize(uint32_t w[8], const f2 gv[8], float r) {
  const f2 rr = make_f2(r, r);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const f2 xv = make_f2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    const f2 y = mul2(mul2(xv, rr), gv[i]);
    w[i] = bf16x2_rn(y.a(), y.b());
  }
}

// Augmented quantization (ARCQuant page, 기술 요약 / 방법론): channels of x
// taken in the order perm, the usual block step on them (primary stage), and
// S appended channels -- the residual e = fma(-q, d, x) of the first S
// reordered channels against the primary stage, quantized with the same block
// step (augment 0), or a copy of them (augment 1, for the weight).  The
// permutation (as byte offsets into a row) and the rows sit in shared memory,
// so the channel gather reads shared memory only.  Each CTA takes p.arc_rows
// rows per step (2 for K up to about 5K channels, 1 for wider rows) through
// p.arc_bufs row buffers (3; 2 above 9K channels, so that two CTAs still fit
// on an SM): the CTA's last warp is the producer, which fills buffer
// s % p.arc_bufs for step s with one bulk copy per row once every
// consumer warp has released it (mbarriers full[] and consumed[]), so the
// consumers run up to p.arc_bufs - 1 steps ahead of the slowest of them with no
// CTA-wide barrier.  Of the consumer threads, the first P own the primary
// block columns t, t + P, ...: a thread reads a column's 16 channel offsets
// once per step and gathers that block from each of the step's rows with
// them.  The remaining ones take the appended blocks (row, j < S/16) of the
// step: each gathers block j again, repeats its primary step and quantizes
// the residual (or copies the codes); kept apart from the primary threads,
// this extra work does not make one warp of every step twice as long as the
// others (a warp's time is that of its slowest lane).  Every wait is bounded:
// one that sees no progress for 4 s records NVFP4_ERR_TIMEOUT, and the
// producer lets the copies it issued land before the CTA exits.
// Output: the [rows, K + S] operand (codes and swizzled scales).
template <bool FOUR_OVER_SIX, int RULE, bool NORM>
__global__ void __launch_bounds__(kArcMaxThreads)
    quantize_arc_kernel(const QuantParams p) {
  BlockConsts k;
  __shared__ ScaleEntry s_dr[128];
  // [K] channel byte offsets, then arc_bufs x [arc_rows][K] rows
  extern __shared__ __align__(16) uint16_t s_dyn[];
  if (!quant_prologue(p, k, s_dr)) return;

  const int64_t K = p.K, KA = p.K + p.S;
  const int R = p.arc_rows;
  const int T = static_cast<int>(blockDim.x), P = p.arc_prim_threads;
  for (int64_t i = threadIdx.x; i < K; i += T) {
    const int32_t c = p.perm[i];
    const int32_t cc = c >= 0 && c < K ? c : 0;  // out-of-range entries read channel 0
    s_dyn[i] = static_cast<uint16_t>(2 * cc);
  }
  const int64_t rows_padded = (p.rows + 127) / 128 * 128;
  const int64_t half_ka = KA / 2, kgroups_a = KA / 64;
  const int nprim = static_cast<int>(K / 16), nres = static_cast<int>(p.S / 16);
  const uint32_t rows_base = smem_u32(s_dyn + K);
  const uint32_t row_bytes = static_cast<uint32_t>(K) * 2, buf_bytes = row_bytes * R;
  // Buffers: full[b] completes when buffer b holds its step's rows (the
  // producer's arrival plus the copies' bytes); consumed[b] when every
  // consumer warp is done with it.  Step s uses buffer s % NB; its waits are
  // on phase s / NB of those barriers.
  const int NB = p.arc_bufs;
  __shared__ __align__(8) uint64_t s_bar[2 * kArcMaxBufs];
  __shared__ int s_abort;
  const uint32_t full0 = smem_u32(&s_bar[0]), consumed0 = smem_u32(&s_bar[kArcMaxBufs]);
  const int warp = static_cast<int>(threadIdx.x >> 5), lane = static_cast<int>(threadIdx.x & 31);
  const int producer_warp = T / 32 - 1;
  if (threadIdx.x == 0) {
    for (int b = 0; b < NB; ++b) {
      mbar_init(full0 + 8 * b, 1);
      mbar_init(consumed0 + 8 * b, producer_warp);  // one arrival per consumer warp
    }
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();  // barriers initialised, channel offsets visible
  volatile int* abort = &s_abort;
  constexpr uint64_t kWaitNs = 4000000000ull;  // no progress for 4 s: report a timeout and stop
  auto fail = [&](uint32_t where) {
    if (!*abort) {
      *abort = 1;
      p.ws->detail = where;
      p.ws->status = NVFP4_ERR_TIMEOUT;
    }
  };
  const int64_t stride_rows = static_cast<int64_t>(gridDim.x) * R;
  if (warp == producer_warp) {
    // ------------------------------------------------------- producer ----
    int s = 0;
    for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * R; row0 < rows_padded; row0 += stride_rows, ++s) {
      const int b = s % NB;
      if (s >= NB && !__all_sync(0xffffffffu, mbar_wait_bounded(consumed0 + 8 * b, (s / NB - 1) & 1, abort, kWaitNs))) {
        if (lane == 0) fail(1);
        break;
      }
      if (lane == 0) {
        const int64_t left = p.rows - row0;
        const int valid = left <= 0 ? 0 : (left < R ? static_cast<int>(left) : R);
        mbar_expect_tx(full0 + 8 * b, static_cast<uint32_t>(valid) * row_bytes);
        for (int rr = 0; rr < valid; ++rr)
          bulk_copy_g2s(rows_base + b * buf_bytes + rr * row_bytes, p.x + (row0 + rr) * p.ldx, row_bytes,
                        full0 + 8 * b);
      }
      __syncwarp();
    }
    if (*abort && lane == 0) {
      // let the copies already issued land before the CTA can exit
      const volatile int no_abort = 0;
      for (int k = s >= NB ? s - NB : 0; k < s; ++k)
        mbar_wait_bounded(full0 + 8 * (k % NB), (k / NB) & 1, &no_abort, 100000000ull);
    }
    return;
  }
  // ---------------------------------------------------------- consumers ----
  auto scale_at = [&](int64_t row, int col) -> uint8_t& {
    return p.scales[(row >> 7) * kgroups_a * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (col >> 2) * 512 +
                    (col & 3)];
  };
  int s = 0;
  for (int64_t row0 = static_cast<int64_t>(blockIdx.x) * R; row0 < rows_padded; row0 += stride_rows, ++s) {
    const int b = s % NB;
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(full0 + 8 * b, (s / NB) & 1, abort, kWaitNs))) {
      if (lane == 0) fail(2);
      break;
    }
    const uint32_t s_buf = rows_base + static_cast<uint32_t>(b) * buf_bytes;  // shared address of the step's rows
    // gather block j of buffer row rr (16 channels as bf16 pairs, element 2i low)
    auto gather = [&](int rr, int j, f2 px[8]) {
      const uint4 o0 = reinterpret_cast<const uint4*>(s_dyn + 16 * j)[0];
      const uint4 o1 = reinterpret_cast<const uint4*>(s_dyn + 16 * j)[1];
      const uint32_t ow[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
      const uint32_t s_row = s_buf + rr * row_bytes;
      uint32_t w[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        w[i] = ld_shared_u16(s_row + (ow[i] & 0xFFFFu)) | (ld_shared_u16(s_row + (ow[i] >> 16)) << 16);
      if (NORM) {
        f2 gv[8];
        rms_gains(p.gperm, j, gv);
        rms_normalize(w, gv, __ldg(p.rinv + row0 + rr));
      }
      return unpack_block(make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4], w[5], w[6], w[7]), px);
    };
    if (static_cast<int>(threadIdx.x) < P) {
      // primary blocks
      for (int j = threadIdx.x; j < nprim; j += P) {
        const uint4 o0 = reinterpret_cast<const uint4*>(s_dyn + 16 * j)[0];
        const uint4 o1 = reinterpret_cast<const uint4*>(s_dyn + 16 * j)[1];
        const uint32_t ow[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        for (int rr = 0; rr < R; ++rr) {
          const int64_t row = row0 + rr;
          uint32_t scale = 0;
          if (row < p.rows) {
            const uint32_t s_row = s_buf + rr * row_bytes;
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              w[i] = ld_shared_u16(s_row + (ow[i] & 0xFFFFu)) | (ld_shared_u16(s_row + (ow[i] >> 16)) << 16);
            if (NORM) {
              // the column's gains, read (L1) and unpacked per row: holding them
              // across the rows takes the registers of a third CTA per SM
              f2 gv[8];
              rms_gains(p.gperm, j, gv);
              rms_normalize(w, gv, __ldg(p.rinv + row));
            }
            f2 px[8];
            const uint32_t bbits = unpack_block(make_uint4(w[0], w[1], w[2], w[3]),
                                                make_uint4(w[4], w[5], w[6], w[7]), px);
            uint2 codes;
            quantize_pairs<FOUR_OVER_SIX, RULE>(px, __uint_as_float(bbits << 16), k, s_dr, codes, scale);
            *reinterpret_cast<uint2*>(p.codes + row * half_ka + j * 8) = codes;
          }
          scale_at(row, j) = static_cast<uint8_t>(scale);
        }
      }
    } else {
      // appended blocks: units (rr, j) of this step, j < S/16
      const int Tr = T - 32 - P;
      for (int u = static_cast<int>(threadIdx.x) - P; u < R * nres; u += Tr) {
        const int rr = u / nres, j = u - rr * nres;
        const int64_t row = row0 + rr;
        uint32_t scale_a = 0;
        if (row < p.rows) {
          f2 px[8];
          const uint32_t bbits = gather(rr, j, px);
          uint2 codes, codes_a;
          uint32_t scale;
          quantize_pairs<FOUR_OVER_SIX, RULE>(px, __uint_as_float(bbits << 16), k, s_dr, codes, scale);
          if (p.augment) {
            codes_a = codes;
            scale_a = scale;
          } else {
            const f2 nd = s_dr[scale].nd;
            f2 q[8], e[8];
            decode_pairs(codes, q);
            float bmax = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              e[i] = fma2(q[i], nd, px[i]);
              bmax = fmaxf(bmax, fmaxf(fabsf(e[i].a()), fabsf(e[i].b())));
            }
            quantize_pairs<FOUR_OVER_SIX, RULE>(e, bmax, k, s_dr, codes_a, scale_a);
          }
          *reinterpret_cast<uint2*>(p.codes + row * half_ka + (nprim + j) * 8) = codes_a;
        }
        scale_at(row, nprim + j) = static_cast<uint8_t>(scale_a);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive_local(consumed0 + 8 * b);  // this warp is done with buffer b
  }
}

// Threads of the augmented quantizer for K channels: P for the primary blocks,
// c block columns each (c >= 2 from 256 columns up, P <= 256, a multiple of
// 32), so that a CTA stays small and several share an SM; then enough for the
// step's R * S/16 appended blocks at about c * R / 2 each (two block steps
// apiece, against c * R for a primary thread), within kArcMaxThreads; at
// least 96 consumers in all; then the producer warp.
int arc_prim_threads(int64_t K) {
  const int64_t nprim = std::max<int64_t>(1, K / 16);
  const int64_t cols = std::max<int64_t>((nprim + kArcPrimThreads - 1) / kArcPrimThreads, nprim >= 256 ? 2 : 1);
  const int64_t t = (nprim + cols - 1) / cols;
  return static_cast<int>((t + 31) / 32 * 32);
}
int arc_threads(int64_t K, int64_t S, int R) {
  const int prim = arc_prim_threads(K);
  const int64_t nprim = std::max<int64_t>(1, K / 16);
  const int64_t cols = (nprim + prim - 1) / prim;
  const int64_t units = R * (S / 16), per = std::max<int64_t>(1, cols * R / 2);
  int64_t res = units == 0 ? 0 : ((units + per - 1) / per + 31) / 32 * 32;
  res = std::min<int64_t>(res, kArcMaxThreads - 32 - prim);  // room for the producer warp
  if (units > 0) res = std::max<int64_t>(res, 32);
  return static_cast<int>(std::max<int64_t>(96, prim + res)) + 32;  // + the producer warp
}

// Rows per step and row buffers of the augmented quantizer for K channels,
// with the K-entry channel offsets ahead of the rows, within kArcSmemStep:
// three buffers of the most rows (up to 4, a power of two so it divides the
// 128-row padding).  Where even one row per buffer does not fit (K above
// about 9K), two buffers of one row (within kArcSmemBudget for K <= 16384), so
// that two CTAs still share an SM.
void arc_layout(int64_t K, int* rows, int* bufs) {
  for (int r = kArcMaxRows; r >= 1; r /= 2) {
    if (2 * K * (1 + kArcMaxBufs * r) <= kArcSmemStep) {
      *rows = r;
      *bufs = kArcMaxBufs;
      return;
    }
  }
  *rows = 1;
  *bufs = 2;
}

template <bool F, int R, bool NORM>
cudaError_t launch_quantize_arc(int dev, int sms, const QuantParams& p, cudaStream_t s, bool pdl) {
  const size_t smem = static_cast<size_t>(p.K) * 2 * (1 + p.arc_bufs * p.arc_rows);
  // the shared-memory opt-in is an attribute of the kernel in this context
  static PerContextCache<int> attr;
  int done = 0;
  cudaError_t e = per_context(attr, dev, [](int* v) {
    *v = 1;
    return cudaFuncSetAttribute(quantize_arc_kernel<F, R, NORM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kArcSmemBudget));
  }, &done);
  if (e != cudaSuccess) return e;
  const int threads = arc_threads(p.K, p.S, p.arc_rows);
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, quantize_arc_kernel<F, R, NORM>, threads, smem);
  if (e != cudaSuccess) return e;
  const int64_t steps = (p.rows + 127) / 128 * 128 / p.arc_rows;
  const int grid = static_cast<int>(std::max<int64_t>(
      1, std::min<int64_t>(steps, static_cast<int64_t>(sms) * std::max(1, occ))));
  return launch_kernel(quantize_arc_kernel<F, R, NORM>, dim3(grid), dim3(threads), smem, s, pdl, p);
}

template <bool NORM>
cudaError_t launch_quantize_arc_norm(int mode, int rule, int dev, int sms, const QuantParams& p, cudaStream_t s,
                                     bool pdl) {
  if (mode == NVFP4_MODE_SIX) return launch_quantize_arc<false, kRuleMax, NORM>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAX) return launch_quantize_arc<true, kRuleMax, NORM>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAE) return launch_quantize_arc<true, kRuleMae, NORM>(dev, sms, p, s, pdl);
  return launch_quantize_arc<true, kRuleMse, NORM>(dev, sms, p, s, pdl);
}

cudaError_t launch_quantize_arc_kernel(int mode, int rule, int dev, int sms, const QuantParams& p,
                                       cudaStream_t s, bool pdl) {
  return p.gamma ? launch_quantize_arc_norm<true>(mode, rule, dev, sms, p, s, pdl)
                 : launch_quantize_arc_norm<false>(mode, rule, dev, sms, p, s, pdl);
}

template <bool F, int R>
cudaError_t launch_quantize_t(int dev, int sms, const QuantParams& p, cudaStream_t s, bool pdl) {
  static PerContextCache<int> per_sm;
  int occ = 0;
  cudaError_t e = per_context(per_sm, dev, [](int* v) {
    const cudaError_t r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, quantize_t_kernel<F, R>, kQuantThreads, 0);
    *v = std::max(1, *v);
    return r;
  }, &occ);
  if (e != cudaSuccess) return e;
  const int64_t tiles = ((p.rows + 127) / 128) * (((p.K + 127) / 128 * 128) / 64);
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(tiles, static_cast<int64_t>(sms) * occ)));
  return launch_kernel(quantize_t_kernel<F, R>, dim3(grid), dim3(kQuantThreads), 0, s, pdl, p);
}

cudaError_t launch_quantize_t_kernel(int mode, int rule, int dev, int sms, const QuantParams& p,
                                     cudaStream_t s, bool pdl) {
  if (mode == NVFP4_MODE_SIX) return launch_quantize_t<false, kRuleMax>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAX) return launch_quantize_t<true, kRuleMax>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAE) return launch_quantize_t<true, kRuleMae>(dev, sms, p, s, pdl);
  return launch_quantize_t<true, kRuleMse>(dev, sms, p, s, pdl);
}

template <bool F, int R, bool V8>
cudaError_t launch_quantize_v(int dev, int sms, const QuantParams& p, cudaStream_t s, bool pdl) {
  static PerContextCache<int> per_sm;
  int occ = 0;
  cudaError_t e = per_context(per_sm, dev, [](int* v) {
    const cudaError_t r =
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, quantize_kernel<F, R, V8>, kQuantThreads, 0);
    *v = std::max(1, *v);
    return r;
  }, &occ);
  if (e != cudaSuccess) return e;
  const int64_t want = (static_cast<int64_t>(p.ntasks) + kQuantWarps - 1) / kQuantWarps;
  const int grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, static_cast<int64_t>(sms) * occ)));
  return launch_kernel(quantize_kernel<F, R, V8>, dim3(grid), dim3(kQuantThreads), 0, s, pdl, p);
}
// 256-bit block loads where every row of x starts on a 32-byte boundary
template <bool F, int R>
cudaError_t launch_quantize(int dev, int sms, const QuantParams& p, cudaStream_t s, bool pdl) {
  const bool v8 = reinterpret_cast<uintptr_t>(p.x) % 32 == 0 && p.ldx % 16 == 0;
  return v8 ? launch_quantize_v<F, R, true>(dev, sms, p, s, pdl) : launch_quantize_v<F, R, false>(dev, sms, p, s, pdl);
}

cudaError_t launch_quantize_kernel(int mode, int rule, int dev, int sms, const QuantParams& p, cudaStream_t s,
                                   bool pdl) {
  if (mode == NVFP4_MODE_SIX) return launch_quantize<false, kRuleMax>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAX) return launch_quantize<true, kRuleMax>(dev, sms, p, s, pdl);
  if (rule == NVFP4_RULE_MAE) return launch_quantize<true, kRuleMae>(dev, sms, p, s, pdl);
  return launch_quantize<true, kRuleMse>(dev, sms, p, s, pdl);
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

size_t nvfp4_quantize_arc_rmsnorm_workspace_bytes(int64_t rows, int64_t K) {
  // the quantize workspace, then 1 / rms of each row, then the gains in channel order
  return nvfp4_quantize_workspace_bytes(rows, K) + align16(sizeof(float) * static_cast<size_t>(rows > 0 ? rows : 0)) +
         align16(sizeof(uint16_t) * static_cast<size_t>(K > 0 ? K : 0));
}

}  // extern "C"

namespace {

// ------------------------------------------------------------ host side --
// Warp tasks of the row-wise kernel: pairs of chunks of 32 blocks of 16
// elements (the last pair of a row may hold one chunk, the last chunk may be
// partial) over the rows padded to a multiple of 128.
int64_t row_tasks(int64_t rows, int64_t K) { return (rows + 127) / 128 * 128 * (((K + 511) / 512 + 1) / 2); }

// Checks shared by every quantize entry point: pointers, shape, row pitch,
// mode, rule, alignment and the size limits of the kernels' index arithmetic.
// `scale_ptr` is the global-scale output (dynamic alpha) or input (static
// alpha).  Row-wise blocks need K a multiple of 64; the transposed form
// (blocks down the columns) needs rows a multiple of 64 and K of 8.
nvfp4_status check_quant_args(const char* fn, bool transposed, const void* x, int64_t rows, int64_t K,
                              int64_t ldx, int mode, int rule, const void* codes, const void* scales,
                              const void* scale_ptr) {
  if (!x || !codes || !scales || !scale_ptr)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  if (!transposed && (rows < 1 || K < 64 || K % 64 != 0))
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "%s: need rows >= 1 and K a positive multiple of 64 (rows=%lld K=%lld)", fn,
                     (long long)rows, (long long)K);
  if (transposed && (rows < 64 || rows % 64 != 0 || K < 8 || K % 8 != 0))
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "%s: need rows a positive multiple of 64 and K a positive multiple of 8 (rows=%lld K=%lld)",
                     fn, (long long)rows, (long long)K);
  if (ldx < K || ldx % 8 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: need ldx >= K and ldx %% 8 == 0", fn);
  if (mode != NVFP4_MODE_SIX && mode != NVFP4_MODE_FOUR_OVER_SIX)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: unknown mode %d", fn, mode);
  if (rule != NVFP4_RULE_MAX && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: unknown rule %d", fn, rule);
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) ||
      (reinterpret_cast<uintptr_t>(scale_ptr) & 3u))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: misaligned buffer", fn);
  // at most 2^40 elements of x (rows * ldx), and a 32-bit warp-task counter
  // in the row-wise kernel
  if (rows > (int64_t{1} << 40) / ldx || row_tasks(rows, K) >= 0x80000000ll)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: tensor too large", fn);
  return NVFP4_OK;
}

nvfp4_status check_fp8_max(const char* fn, float fp8_max) {
  if (!(fp8_max == 448.0f || fp8_max == 256.0f))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: fp8_max must be 448 or 256", fn);
  return NVFP4_OK;
}

// CTAs of the amax pass: enough for eight 16-byte loads per thread, at most
// two per SM (dense x), or one per row up to two per SM (pitched x).
int amax_grid_size(int64_t rows, int64_t K, int64_t ldx, int sms) {
  int64_t g;
  if (ldx == K)
    g = std::min<int64_t>((rows * K / 8 + kAmaxThreads * 8 - 1) / (kAmaxThreads * 8), int64_t{sms} * 2);
  else
    g = std::min<int64_t>(rows, int64_t{sms} * 2);
  return static_cast<int>(std::max<int64_t>(1, g));
}

// Kernel parameters common to every entry point; the caller sets the alpha
// source (partials + nparts + f6 and global_scale, or alpha_in).
QuantParams base_params(const void* x, int64_t rows, int64_t K, int64_t ldx, void* codes, void* scales,
                        WorkspaceHeader* ws) {
  QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.rows = rows;
  p.K = K;
  p.ldx = ldx;
  p.codes = static_cast<uint8_t*>(codes);
  p.scales = static_cast<uint8_t*>(scales);
  p.global_scale = nullptr;
  p.partials = nullptr;
  p.alpha_in = nullptr;
  p.ws = ws;
  p.nparts = 0;
  p.f6 = 0.0f;
  p.ntasks = static_cast<uint32_t>(row_tasks(rows, K));
  p.chunks = static_cast<uint32_t>((K + 511) / 512);
  p.kgroups = static_cast<uint32_t>(K / 64);
  return p;
}

// The amax pass into `partials` (amax_grid CTAs), then the quantize kernel
// of `kind` with alpha reduced from those partials.
enum class QuantKind { kRows, kTransposed, kAugmented };

nvfp4_status launch_dynamic(QuantKind kind, QuantParams p, int mode, int rule, float fp8_max,
                            float* global_scale, uint32_t* partials, int amax_grid, int dev, int sms,
                            cudaStream_t s) {
  amax_kernel<<<amax_grid, kAmaxThreads, 0, s>>>(p.x, p.rows, p.K, p.ldx, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_status(e, "amax_kernel launch");
  p.global_scale = global_scale;
  p.partials = partials;
  p.nparts = amax_grid;
  p.f6 = fp8_max * 6.0f;
  // the quantize kernel is a programmatic dependent of the amax pass: it is
  // scheduled while the amax pass drains and waits for it in its prologue
  e = kind == QuantKind::kTransposed ? launch_quantize_t_kernel(mode, rule, dev, sms, p, s, true)
      : kind == QuantKind::kAugmented ? launch_quantize_arc_kernel(mode, rule, dev, sms, p, s, true)
                                       : launch_quantize_kernel(mode, rule, dev, sms, p, s, true);
  if (e != cudaSuccess) return cuda_status(e, "quantize kernel launch");
  return NVFP4_OK;
}

// The RMS pass, then the augmented quantizer with RMSNorm as its
// programmatic dependent.
// One wave of CTAs of `kernel` (threads each), at most one warp per row.
template <typename Kernel>
cudaError_t rms_grid(PerContextCache<int>& per_sm, Kernel kernel, int threads, int dev, int sms, int64_t rows,
                     int* grid) {
  int occ = 0;
  const cudaError_t e = per_context(per_sm, dev, [kernel, threads](int* v) {
    const cudaError_t r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(v, kernel, threads, 0);
    *v = std::max(1, *v);
    return r;
  }, &occ);
  if (e != cudaSuccess) return e;
  const int64_t want = (rows + threads / 32 - 1) / (threads / 32);
  *grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(want, int64_t{sms} * occ),
                                                                  kMaxPartials)));
  return cudaSuccess;
}

template <int NR, bool V8>
cudaError_t launch_rms_reg_v(const QuantParams& p, uint32_t* partials, float eps, int dev, int sms, cudaStream_t s,
                             int* grid) {
  static PerContextCache<int> per_sm;
  cudaError_t e = rms_grid(per_sm, rms_amax_reg_kernel<NR, V8>, kRmsRegThreads, dev, sms, p.rows, grid);
  if (e != cudaSuccess) return e;
  rms_amax_reg_kernel<NR, V8><<<*grid, kRmsRegThreads, 0, s>>>(p.x, p.rows, p.K, p.ldx, p.gamma, eps, p.perm,
                                                            const_cast<float*>(p.rinv),
                                                            const_cast<uint16_t*>(p.gperm), partials);
  return cudaGetLastError();
}
// 256-bit loads where x's rows and the gains start on 32-byte boundaries
bool rms_aligned32(const QuantParams& p) {
  return reinterpret_cast<uintptr_t>(p.x) % 32 == 0 && p.ldx % 16 == 0 &&
         reinterpret_cast<uintptr_t>(p.gamma) % 32 == 0;
}
template <int NR>
cudaError_t launch_rms_reg(const QuantParams& p, uint32_t* partials, float eps, int dev, int sms, cudaStream_t s,
                           int* grid) {
  return rms_aligned32(p) ? launch_rms_reg_v<NR, true>(p, partials, eps, dev, sms, s, grid)
                          : launch_rms_reg_v<NR, false>(p, partials, eps, dev, sms, s, grid);
}
template <bool V8>
cudaError_t launch_rms_stream(const QuantParams& p, uint32_t* partials, float eps, int dev, int sms, cudaStream_t s,
                              int* grid) {
  static PerContextCache<int> per_sm;
  cudaError_t e = rms_grid(per_sm, rms_amax_kernel<V8>, kRmsThreads, dev, sms, p.rows, grid);
  if (e != cudaSuccess) return e;
  rms_amax_kernel<V8><<<*grid, kRmsThreads, 0, s>>>(p.x, p.rows, p.K, p.ldx, p.gamma, eps, p.perm,
                                                   const_cast<float*>(p.rinv), const_cast<uint16_t*>(p.gperm),
                                                   partials);
  return cudaGetLastError();
}

cudaError_t launch_rms_pass(const QuantParams& p, uint32_t* partials, float eps, int dev, int sms, cudaStream_t s,
                            int* grid) {
  // the row in registers up to K = 8192 (168 registers at 8 rounds), round by
  // round above that
  switch ((p.K + 1023) / 1024) {
    case 1: return launch_rms_reg<1>(p, partials, eps, dev, sms, s, grid);
    case 2: return launch_rms_reg<2>(p, partials, eps, dev, sms, s, grid);
    case 3: return launch_rms_reg<3>(p, partials, eps, dev, sms, s, grid);
    case 4: return launch_rms_reg<4>(p, partials, eps, dev, sms, s, grid);
    case 5: return launch_rms_reg<5>(p, partials, eps, dev, sms, s, grid);
    case 6: return launch_rms_reg<6>(p, partials, eps, dev, sms, s, grid);
    case 7: return launch_rms_reg<7>(p, partials, eps, dev, sms, s, grid);
    case 8: return launch_rms_reg<8>(p, partials, eps, dev, sms, s, grid);
    default: break;
  }
  return rms_aligned32(p) ? launch_rms_stream<true>(p, partials, eps, dev, sms, s, grid)
                          : launch_rms_stream<false>(p, partials, eps, dev, sms, s, grid);
}

nvfp4_status launch_rms_dynamic(QuantParams p, int mode, int rule, float fp8_max, float* global_scale,
                                uint32_t* partials, float eps, int dev, int sms, cudaStream_t s) {
  int grid = 0;
  cudaError_t e = launch_rms_pass(p, partials, eps, dev, sms, s, &grid);
  if (e != cudaSuccess) return cuda_status(e, "RMS pass launch");
  p.global_scale = global_scale;
  p.partials = partials;
  p.nparts = grid;
  p.f6 = fp8_max * 6.0f;
  e = launch_quantize_arc_kernel(mode, rule, dev, sms, p, s, true);
  if (e != cudaSuccess) return cuda_status(e, "quantize kernel launch");
  return NVFP4_OK;
}

// nvfp4_quantize (row-wise blocks of x), nvfp4_quantize_t (blocks along the
// rows of x, i.e. the operand of x^T) and nvfp4_quantize_arc (row-wise with
// reordered and augmented channels), with the caller's workspace.
// Every host-side argument check of a dynamic-alpha quantize call (not the
// device check); enqueues nothing.
nvfp4_status check_quantize_call(const char* fn, QuantKind kind, const void* x, int64_t rows, int64_t K,
                                 int64_t ldx, int mode, int rule, float fp8_max, const void* codes,
                                 const void* scales, const float* global_scale, const void* workspace,
                                 size_t workspace_bytes, const int32_t* perm, int64_t S, int augment,
                                 const uint16_t* gamma = nullptr, float eps = 0.0f) {
  nvfp4_status st = check_quant_args(fn, kind == QuantKind::kTransposed, x, rows, K, ldx, mode, rule, codes,
                                     scales, global_scale);
  if (st != NVFP4_OK) return st;
  if ((st = check_fp8_max(fn, fp8_max)) != NVFP4_OK) return st;
  if (kind == QuantKind::kAugmented) {
    if (!perm || (reinterpret_cast<uintptr_t>(perm) & 3u))
      return set_error(NVFP4_ERR_INVALID_ARG, "%s: perm must be a non-null 4-byte aligned device pointer", fn);
    if (S < 0 || S % 64 != 0 || S > K)
      return set_error(NVFP4_ERR_INVALID_ARG, "%s: need 0 <= S <= K and S %% 64 == 0 (S=%lld)", fn, (long long)S);
    if (K > kArcMaxK) return set_error(NVFP4_ERR_INVALID_ARG, "%s: K above %lld", fn, (long long)kArcMaxK);
    if (augment != 0 && augment != 1) return set_error(NVFP4_ERR_INVALID_ARG, "%s: augment must be 0 or 1", fn);
  }
  if (!workspace || !aligned16(workspace))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace must be a non-null 16-byte aligned pointer", fn);
  if (gamma) {
    if (!aligned16(gamma)) return set_error(NVFP4_ERR_INVALID_ARG, "%s: gamma must be 16-byte aligned", fn);
    if (!(eps > 0.0f) || isinf(eps))
      return set_error(NVFP4_ERR_INVALID_ARG, "%s: eps must be a positive finite number", fn);
    if (workspace_bytes < nvfp4_quantize_arc_rmsnorm_workspace_bytes(rows, K))
      return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace too small", fn);
  }
  if (workspace_bytes < nvfp4_quantize_workspace_bytes(rows, K))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace too small", fn);
  return NVFP4_OK;
}

nvfp4_status quantize_impl(const char* fn, QuantKind kind, const void* x, int64_t rows, int64_t K,
                           int64_t ldx, int mode, int rule, float fp8_max, void* codes, void* scales,
                           float* global_scale, void* workspace, size_t workspace_bytes, void* stream,
                           const int32_t* perm = nullptr, int64_t S = 0, int augment = 0,
                           const uint16_t* gamma = nullptr, float eps = 0.0f) {
  nvfp4_status st = check_quantize_call(fn, kind, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                                        global_scale, workspace, workspace_bytes, perm, S, augment, gamma, eps);
  if (st != NVFP4_OK) return st;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != NVFP4_OK) return st;

  auto* ws = static_cast<WorkspaceHeader*>(workspace);
  auto* partials = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + sizeof(WorkspaceHeader));
  QuantParams p = base_params(x, rows, K, ldx, codes, scales, ws);
  p.perm = perm;
  p.S = S;
  p.augment = augment;
  if (kind == QuantKind::kAugmented) {
    arc_layout(K, &p.arc_rows, &p.arc_bufs);
    p.arc_prim_threads = arc_prim_threads(K);
  }
  if (gamma) {
    // RMSNorm ahead of the augmented quantizer: the RMS pass takes the amax
    // pass's place and leaves 1/rms of every row after the partials
    p.gamma = gamma;
    p.rinv = reinterpret_cast<float*>(static_cast<char*>(workspace) + nvfp4_quantize_workspace_bytes(rows, K));
    p.gperm = reinterpret_cast<const uint16_t*>(static_cast<char*>(workspace) + nvfp4_quantize_workspace_bytes(rows, K) +
                                                 align16(sizeof(float) * static_cast<size_t>(rows)));
    return launch_rms_dynamic(p, mode, rule, fp8_max, global_scale, partials, eps, dev, sms,
                              static_cast<cudaStream_t>(stream));
  }
  const int amax_grid = std::min(amax_grid_size(rows, K, ldx, sms), kMaxPartials);
  return launch_dynamic(kind, p, mode, rule, fp8_max, global_scale, partials, amax_grid, dev, sms,
                        static_cast<cudaStream_t>(stream));
}

}  // namespace

namespace nvfp4 {

nvfp4_status quantize_rows_check(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                                 int rule, float fp8_max, const void* codes, const void* scales,
                                 const float* global_scale, const void* workspace, size_t workspace_bytes) {
  return check_quantize_call(fn, QuantKind::kRows, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                             global_scale, workspace, workspace_bytes, nullptr, 0, 0);
}

nvfp4_status quantize_arc_check(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx,
                                const int32_t* perm, int64_t S, int augment, int mode, int rule, float fp8_max,
                                const void* codes, const void* scales, const float* global_scale,
                                const void* workspace, size_t workspace_bytes, const void* gamma, float eps) {
  return check_quantize_call(fn, QuantKind::kAugmented, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                             global_scale, workspace, workspace_bytes, perm, S, augment,
                             static_cast<const uint16_t*>(gamma), eps);
}

nvfp4_status quantize_arc_enqueue(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx,
                                  const int32_t* perm, int64_t S, int augment, int mode, int rule, float fp8_max,
                                  void* codes, void* scales, float* global_scale, void* workspace,
                                  size_t workspace_bytes, void* stream, const void* gamma, float eps) {
  return quantize_impl(fn, QuantKind::kAugmented, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                       global_scale, workspace, workspace_bytes, stream, perm, S, augment,
                       static_cast<const uint16_t*>(gamma), eps);
}

nvfp4_status quantize_rows_enqueue(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                                   int rule, float fp8_max, void* codes, void* scales, float* global_scale,
                                   void* workspace, size_t workspace_bytes, void* stream) {
  return quantize_impl(fn, QuantKind::kRows, x, rows, K, ldx, mode, rule, fp8_max, codes, scales, global_scale,
                       workspace, workspace_bytes, stream);
}

}  // namespace nvfp4

extern "C" {

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                            int rule, float fp8_max, void* codes, void* scales,
                            float* global_scale, void* workspace, size_t workspace_bytes,
                            void* stream) {
  return quantize_impl("nvfp4_quantize", QuantKind::kRows, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                       global_scale, workspace, workspace_bytes, stream);
}

nvfp4_status nvfp4_quantize_arc(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                const int32_t* perm, int64_t S, int augment, int mode, int rule,
                                float fp8_max, void* codes, void* scales, float* global_scale,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return quantize_impl("nvfp4_quantize_arc", QuantKind::kAugmented, x, rows, K, ldx, mode, rule, fp8_max,
                       codes, scales, global_scale, workspace, workspace_bytes, stream, perm, S, augment);
}

nvfp4_status nvfp4_quantize_arc_rmsnorm(const void* x, int64_t rows, int64_t K, int64_t ldx, const void* gamma,
                                        float eps, const int32_t* perm, int64_t S, int mode, int rule,
                                        float fp8_max, void* codes, void* scales, float* global_scale,
                                        void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "nvfp4_quantize_arc_rmsnorm";
  if (!gamma) return set_error(NVFP4_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  return quantize_impl(fn, QuantKind::kAugmented, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                       global_scale, workspace, workspace_bytes, stream, perm, S, 0,
                       static_cast<const uint16_t*>(gamma), eps);
}

nvfp4_status nvfp4_quantize_t(const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                              int rule, float fp8_max, void* codes, void* scales,
                              float* global_scale, void* workspace, size_t workspace_bytes,
                              void* stream) {
  return quantize_impl("nvfp4_quantize_t", QuantKind::kTransposed, x, rows, K, ldx, mode, rule, fp8_max, codes, scales,
                       global_scale, workspace, workspace_bytes, stream);
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
// CTAs (the launch uses at most 2 per SM, 296 on a B200); a launch that would
// need more is rejected.  Nothing in it has to start at zero: each call's amax
// kernel writes every partial slot the following quantize kernel reads, and
// the quantize kernel writes the status word.  All calls on a device share it,
// so two calls that may overlap on the GPU (different streams without an
// ordering between them) race on it and must be serialized by the caller.

namespace nvfp4 {
namespace {

constexpr size_t kNoAllocScratchBytes = sizeof(WorkspaceHeader) + sizeof(uint32_t) * kMaxPartials;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

static PerContextCache<void*> g_noalloc_addr;

// Device address of g_noalloc_scratch on the current device `dev`, looked up
// with that device current once per CUDA context: the first call on a device
// does this set-up, and so does the first call after the device's context
// was reset or replaced (the module, and with it the array, is loaded anew).
// In host code the array's name is only a host-side stand-in for the symbol,
// never a device address, so kernels must get this pointer instead.
nvfp4_status noalloc_scratch(int dev, void** out) {
  cudaError_t e = per_context(g_noalloc_addr, dev, [](void** p) {
    return cudaGetSymbolAddress(p, g_noalloc_scratch);
  }, out);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetSymbolAddress(noalloc scratch)");
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                               int mode, int rule, float fp8_max, void* codes,
                                               void* scales, float* global_scale, void* stream) {
  const char* fn = "nvfp4_quantize_noalloc";
  nvfp4_status st = check_quant_args(fn, false, x, rows, K, ldx, mode, rule, codes, scales, global_scale);
  if (st != NVFP4_OK) return st;
  if ((st = check_fp8_max(fn, fp8_max)) != NVFP4_OK) return st;
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != NVFP4_OK) return st;
  const int amax_grid = amax_grid_size(rows, K, ldx, sms);
  if (amax_grid > kMaxPartials)
    return set_error(NVFP4_ERR_INVALID_ARG,
                     "%s: the amax pass needs %d partial slots but the static scratch holds %d (%zu bytes)", fn,
                     amax_grid, kMaxPartials, kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((st = noalloc_scratch(dev, &scratch)) != NVFP4_OK) return st;
  auto* ws = static_cast<WorkspaceHeader*>(scratch);
  auto* partials = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + sizeof(WorkspaceHeader));
  return launch_dynamic(QuantKind::kRows, base_params(x, rows, K, ldx, codes, scales, ws), mode, rule, fp8_max,
                        global_scale, partials, amax_grid, dev, sms, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------ static tensor scale --
// nvfp4_quantize with a caller-supplied alpha (e.g. calibrated offline): the
// amax pass and its HBM read of x are skipped, one kernel launch.

extern "C" nvfp4_status nvfp4_quantize_with_scale(const void* x, int64_t rows, int64_t K, int64_t ldx,
                                                  int mode, int rule, const float* global_scale,
                                                  void* codes, void* scales, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
  const char* fn = "nvfp4_quantize_with_scale";
  nvfp4_status st = check_quant_args(fn, false, x, rows, K, ldx, mode, rule, codes, scales, global_scale);
  if (st != NVFP4_OK) return st;
  if (!workspace || !aligned16(workspace))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace must be a non-null 16-byte aligned pointer", fn);
  if (workspace_bytes < sizeof(WorkspaceHeader))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace too small", fn);
  int dev = 0, sms = 0;
  if ((st = check_device(&dev, &sms)) != NVFP4_OK) return st;
  QuantParams p = base_params(x, rows, K, ldx, codes, scales, static_cast<WorkspaceHeader*>(workspace));
  p.alpha_in = global_scale;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, 2 * sizeof(uint32_t), s);  // status, detail
  if (e != cudaSuccess) return cuda_status(e, "nvfp4_quantize_with_scale: status reset");
  e = launch_quantize_kernel(mode, rule, dev, sms, p, s, false);
  if (e != cudaSuccess) return cuda_status(e, "quantize_kernel launch");
  return NVFP4_OK;
}
