// gemm.cu -- NVFP4 x NVFP4 GEMM (W4A4 linear layer) on the sm_100a fifth-
// generation tensor cores.
//
// Y[m, n] = (alpha_A * alpha_B) * sum_kb sA[m,kb] sB[n,kb] sum_{k in kb} qA[m,k] qB[n,k]
// for operands quantized as in nvfp4_quantize: E2M1 codes (two per byte,
// K-major) and one E4M3 scale per 16 elements along K (ARCQuant summary,
// gist.science/ko/paper/2601.07475, "방법론": one uniform NVFP4 GEMM along K;
// Minima page "심층 분석": per-tensor global scales applied around the fused
// GEMM).
//
// Kernel shape: persistent CTA pairs (clusters of 2 on neighbouring SMs), each
// pair walking 256 x 256 output tiles (tile t, t + pairs, ...).  The pair
// issues one tcgen05.mma.cta_group::2 (M=256, N=256, K=64) per K step: CTA r
// holds rows [128r, 128r+128) of the A tile and the same half of the B tile
// in its shared memory, and the accumulator rows [128r, 128r+128) x 256 in
// its TMEM, so every operand byte crosses each SM's shared memory once.
// K is consumed 256 elements (128 bytes per row) per stage through a 5-stage
// ring that runs on across tile boundaries.
//   warp 0      TMA producer (both CTAs): A half 128x128 B and B half 128x128 B
//               (128-byte swizzle) plus the K step's scale atoms (3-D tensor
//               maps over the swizzled scale buffers: this CTA's 128-row A
//               atoms, both 128-row B atoms); all of them complete on the
//               leader CTA's stage barrier.  Out-of-range rows, columns and
//               K groups are zero-filled by the tensor maps.
//   warp 1      TMEM allocation (pair) and, in the leader CTA only, the MMA
//               issuer: per K step one tcgen05.cp.cta_group::2 of the A scale
//               atom and two of the B atoms into TMEM (replicated over the
//               four 32-lane subpartitions), then that K step's MMA; commits
//               free the stage in both CTAs and finally the accumulator.  The whole
//               warp runs the loop converged and one elected lane issues each
//               tcgen05 instruction (issuing them from a lone lane of a
//               diverged warp is several times slower).
//   warps 2..5  epilogue (both CTAs): per 64-column subtile, tcgen05.ld of 32
//               lanes x 64 columns, multiply by alpha_A*alpha_B, convert,
//               write the 32 x 128-byte block to a staging buffer in shared
//               memory (128-byte swizzle) and TMA-store it (two buffers per
//               warp, bulk-group waits before reuse); when Y's base or row
//               pitch is not 16-byte aligned, direct stores of one row per lane.
// TMEM (512 columns per CTA): two accumulators that share one 64-column
// subtile, buffer 0 = columns 0..255 and buffer 1 = columns 192..447, and
// one stage of scales at 448..495 (per K step: 4 columns of A scales, 8 of B
// scales); the copies and MMAs of one thread execute in order, so a single
// buffer suffices.  The epilogue loads the shared columns 192..255 first,
// releases them to the next tile's MMAs at once, and stores the rest of tile
// i while the mainloop of tile i+1 runs.
// Every wait is bounded: a wait that makes no progress for the timeout (4 s
// by default, on %globaltimer) records NVFP4_ERR_TIMEOUT in the workspace,
// raises a CTA-wide abort flag, and every role drains what it has in flight
// before TMEM is freed.  The bound is per wait, so a long GEMM whose waits
// keep completing never times out.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "block_step.cuh"
#include "common.cuh"
#include "nvfp4_testing.h"

namespace nvfp4 {
namespace {

constexpr int BM = 256;                 // rows per pair tile (128 per CTA)
constexpr int BN = 256;                 // columns per pair tile
constexpr int HALF = 128;               // rows of A and of B held per CTA
constexpr int BK_BYTES = 128;           // 256 FP4 elements per row per stage
constexpr int STAGES = 5;
constexpr int kThreads = 192;                  // 6 warps
constexpr uint32_t A_STAGE = HALF * BK_BYTES;  // 16 KB
constexpr uint32_t B_STAGE = HALF * BK_BYTES;  // 16 KB
constexpr uint32_t SFA_STAGE = 4 * 512;        // 4 atoms (4 K-groups x 128 rows)
constexpr uint32_t SFB_STAGE = 2 * 4 * 512;    // [row block 0..1][K-group 0..3]
constexpr uint32_t STAGE_TX = A_STAGE + B_STAGE + SFA_STAGE + SFB_STAGE;  // per CTA
constexpr uint32_t OFF_A = 0;
constexpr uint32_t OFF_B = OFF_A + STAGES * A_STAGE;
constexpr uint32_t OFF_SFA = OFF_B + STAGES * B_STAGE;
constexpr uint32_t OFF_SFB = OFF_SFA + STAGES * SFA_STAGE;
constexpr uint32_t OFF_BAR = OFF_SFB + STAGES * SFB_STAGE;
// full[], empty[], acc_full, acc_free, drain
constexpr uint32_t NUM_BARS = 2 * STAGES + 3;
constexpr uint32_t OFF_MISC = OFF_BAR + NUM_BARS * 8;
// epilogue staging for TMA stores: per epilogue warp two 32-row x 128-byte
// buffers (1024-byte aligned for the 128-byte swizzle)
constexpr uint32_t STG_BYTES = 32 * 128;
constexpr uint32_t OFF_STG = (OFF_MISC + 16 + 1023) & ~1023u;
constexpr uint32_t SMEM_BYTES = OFF_STG + 4 * 2 * STG_BYTES + 1024;  // + alignment slack
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t EPI_N = 64;                    // epilogue subtile (columns)
constexpr uint32_t TM_ACC1 = 256 - EPI_N;         // buffer 1 starts on buffer 0's last subtile
constexpr uint32_t TM_SF = TM_ACC1 + 256;         // 448: scales
constexpr uint32_t TM_SFA = TM_SF;                // 4 columns per K step
constexpr uint32_t TM_SFB = TM_SF + 16;           // 8 columns per K step
static_assert(TM_SFB + 32 <= TMEM_COLS, "scales must fit after the accumulators");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");
static_assert(2 * STAGE_TX < (1u << 20), "transaction count range of an mbarrier phase");

// Instruction descriptor, kind::mxf4nvf4: A/B format E2M1 (1) at bits 7-9 and
// 10-12, K-major A and B, N>>3 at bits 17-22, scale format UE4M3 (0) at bit
// 23, M>>4 at bits 24-28 (M = 256 across the CTA pair), dense K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) | (uint32_t(BM >> 4) << 24);

// Shared-memory matrix descriptor for a K-major operand tile written by TMA
// with the 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart
// (SBO), descriptor version 1, layout type 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t operand_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}
// Descriptor of one 512-byte scale atom for tcgen05.cp 32x128b: 32 rows of
// 16 bytes, no swizzle, 8-row core matrices 128 bytes apart (SBO).
__device__ __forceinline__ uint64_t scale_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(128 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46);
}

// Copies one 128-row scale atom from each CTA's shared memory (same offset)
// into each CTA's TMEM, replicated over the four 32-lane subpartitions.
__device__ __forceinline__ void tmem_copy_scales_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

__device__ __forceinline__ void mma_nvf4_pair(uint32_t tacc, uint64_t adesc, uint64_t bdesc,
                                              uint32_t tsfa, uint32_t tsfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          tacc),
      "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

constexpr int kMaxSegments = 16;

struct GemmParams {
  const float* a_global;
  const float* b_global;  // nseg entries: alpha_B of each output-column segment
  int nseg;
  int seg_end[kMaxSegments];  // exclusive end column of each segment; the last is N
  void* y;
  WorkspaceHeader* ws;
  int64_t ldy;
  int M, N;
  uint32_t kgroups;       // K / 64
  uint32_t ktiles;        // ceil(K / 256)
  uint32_t n_tiles;       // ceil(N / 256)
  uint32_t m_tiles;       // ceil(M / 256)
  uint32_t num_tiles;     // ceil(M / 256) * n_tiles
  int out_fp32;
  int vec_store;          // rows of Y start 16-byte aligned: vector stores
  int tma_store;          // Y base and row pitch 16-byte aligned: TMA stores through shared memory
  // NVFP4 output (epilogue kinds 1..4): Y quantized with a caller-supplied alpha
  const float* q_alpha;
  uint8_t* q_codes;       // [M, N/2]
  uint8_t* q_scales;      // swizzled, nvfp4_scales_bytes(M, N)
  uint64_t timeout_ns;
  int debug_flags;        // bit 0: never issue the first stage's copies (timeout test)
};

// Tile order: groups of kTileGroupM rows of output tiles, group by group;
// inside a group the tile row (M) index advances fastest, then the tile
// column.  The tiles in flight at once then share a few A row panels and B
// column panels (measured 3 % faster on the prefill GEMM than an ungrouped
// column-fastest order, with half the DRAM re-reads of B).
constexpr uint32_t kTileGroupM = 32;
__device__ __forceinline__ void tile_origin(const GemmParams& p, uint32_t tile, int& m0, int& n0) {
  const uint32_t span = kTileGroupM * p.n_tiles, grp = tile / span, in_g = tile - grp * span;
  const uint32_t first_m = grp * kTileGroupM, gm = min(kTileGroupM, p.m_tiles - first_m);
  m0 = static_cast<int>(first_m + in_g % gm) * BM;
  n0 = static_cast<int>(in_g / gm) * BN;
}

__device__ __forceinline__ void record_timeout(const GemmParams& p, volatile int* abort,
                                               uint32_t where) {
  *abort = 1;
  p.ws->detail = where;
  p.ws->status = NVFP4_ERR_TIMEOUT;
}

// EPI: 0 = bf16 / fp32 output; 1 = NVFP4 output, scale-6; 2, 3, 4 = NVFP4
// output, Four-Over-Six with the max / MAE / MSE rule.
template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar_full = sbase + OFF_BAR;
  const uint32_t bar_empty = bar_full + 8 * STAGES;
  const uint32_t bar_acc_full = bar_empty + 8 * STAGES;
  const uint32_t bar_acc_free = bar_acc_full + 8;
  const uint32_t bar_drain = bar_acc_free + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();          // 0 = leader (issues the MMAs)
  const uint32_t pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);   // the leader's expect_tx arrival (+ both CTAs' bytes)
      mbar_init(bar_empty + 8 * s, 1);  // the leader's MMA commit
    }
    mbar_init(bar_acc_full, 1);
    mbar_init(bar_acc_free, 8);  // one arrive per epilogue warp of both CTAs
    mbar_init(bar_drain, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSFA);
    prefetch_tensormap(&tmSFB);
    if (p.tma_store) prefetch_tensormap(&tmY);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // launched as a programmatic dependent of the quantize kernel that writes
  // A: everything above overlapped that kernel's tail; no global memory is
  // touched before it has finished
  pdl_wait();

  if (warp == 0) {
    // -------------------------------------------------- TMA producer ----
    // The whole warp walks the loop; one elected lane issues.
    uint32_t it = 0;  // k-step counter across this pair's tiles
    // B (the weight) is re-read by every row of output tiles: keep it in L2
    const uint64_t pol_keep = l2_policy_evict_last();
    bool stop = false;
    for (uint32_t tile = pair; tile < p.num_tiles && !stop; tile += npairs) {
      int m0, n0;
      tile_origin(p, tile, m0, n0);
      const int a_row = m0 + static_cast<int>(rank) * HALF;
      const int b_row = n0 + static_cast<int>(rank) * HALF;
      for (uint32_t kt = 0; kt < p.ktiles; ++kt, ++it) {
        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
        if (it >= STAGES &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(bar_empty + 8 * s, ph ^ 1u, abort, p.timeout_ns))) {
          if (lane == 0 && !*abort) record_timeout(p, abort, 1);
          stop = true;
          break;
        }
        if (elect_one()) {
          const uint32_t fb = map_to_rank(bar_full + 8 * s, 0);  // the leader's stage barrier
          if (rank == 0) mbar_expect_tx(bar_full + 8 * s, 2 * STAGE_TX);
          if (!((p.debug_flags & 1) && it == 0)) {  // test hook: the first stage never fills
            const int32_t kx = static_cast<int32_t>(kt * BK_BYTES);
            tma_load_2d_pair(sbase + OFF_A + s * A_STAGE, &tmA, fb, kx, a_row);
            tma_load_2d_pair_hint(sbase + OFF_B + s * B_STAGE, &tmB, fb, kx, b_row, pol_keep);
            tma_load_3d_pair(sbase + OFF_SFA + s * SFA_STAGE, &tmSFA, fb, 0,
                             static_cast<int32_t>(kt * 4), a_row / 128);
            tma_load_3d_pair_hint(sbase + OFF_SFB + s * SFB_STAGE, &tmSFB, fb, 0,
                                  static_cast<int32_t>(kt * 4), n0 / 128, pol_keep);
          }
        }
        __syncwarp();
      }
    }
    if (*abort && lane == 0) {
      // Drain: let the copies this CTA issued for its last stages land
      // before the CTA can exit.  The leader watches its stage barriers
      // (they complete once both CTAs' bytes arrived); the other CTA, whose
      // copies complete on the leader's barriers, waits out a 2 ms grace
      // period instead -- a bulk copy of a few KB lands in microseconds.
      if (rank == 0) {
        const volatile int no_abort = 0;
        const uint32_t first = it > STAGES ? it - STAGES : 0;
        for (uint32_t k = first; k < it; ++k)
          mbar_wait_bounded(bar_full + 8 * (k % STAGES), (k / STAGES) & 1u, &no_abort, 100000000ull);
      } else {
        const uint64_t now = global_timer_ns();
        while (global_timer_ns() < now + 2000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // ------------------------------------------------ MMA issuer ------
      // The whole warp walks the loop; one elected lane issues.
      const uint32_t own_empty = map_to_rank(bar_empty, 0);
      const uint32_t peer_empty = map_to_rank(bar_empty, 1);
      const uint32_t acc_full_0 = map_to_rank(bar_acc_full, 0);
      const uint32_t acc_full_1 = map_to_rank(bar_acc_full, 1);
      bool any_mma = false, stop = false;
      uint32_t it = 0, local = 0;
      for (uint32_t tile = pair; tile < p.num_tiles && !stop; tile += npairs, ++local) {
        // The accumulator this tile writes overlaps the previous tile's
        // first-drained subtiles: wait until both CTAs' epilogues released them.
        if (local > 0 &&
            !__all_sync(0xffffffffu, mbar_wait_bounded(bar_acc_free, (local - 1) & 1u, abort, p.timeout_ns))) {
          if (lane == 0 && !*abort) record_timeout(p, abort, 4);
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + ((local & 1u) ? TM_ACC1 : 0u);
        for (uint32_t kt = 0; kt < p.ktiles; ++kt, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_full + 8 * s, ph, abort, p.timeout_ns))) {
            if (lane == 0 && !*abort) record_timeout(p, abort, 2);
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t nk = min(4u, p.kgroups - kt * 4);
          const uint32_t sfa = sbase + OFF_SFA + s * SFA_STAGE;
          const uint32_t sfb = sbase + OFF_SFB + s * SFB_STAGE;
          const uint32_t sa = sbase + OFF_A + s * A_STAGE;
          const uint32_t sb = sbase + OFF_B + s * B_STAGE;
          if (elect_one()) {
            // Each K step's scale copies go right before its MMA: an MMA
            // waits for the copies issued ahead of it, while copies issued
            // after an MMA run alongside it.
            for (uint32_t j = 0; j < nk; ++j) {
              tmem_copy_scales_pair(tmem + TM_SFA + 4 * j, scale_desc(sfa + 512 * j));
              tmem_copy_scales_pair(tmem + TM_SFB + 8 * j, scale_desc(sfb + 512 * j));
              tmem_copy_scales_pair(tmem + TM_SFB + 8 * j + 4, scale_desc(sfb + 2048 + 512 * j));
              mma_nvf4_pair(acc, operand_desc(sa + 32 * j), operand_desc(sb + 32 * j),
                            tmem + TM_SFA + 4 * j, tmem + TM_SFB + 8 * j, (kt | j) != 0);
            }
            tc_commit_pair(own_empty + 8 * s);
            tc_commit_pair(peer_empty + 8 * s);
          }
          __syncwarp();
          any_mma = true;
        }
        if (!stop && elect_one()) {
          tc_commit_pair(acc_full_0);
          tc_commit_pair(acc_full_1);
        }
        __syncwarp();
      }
      const bool drain = __shfl_sync(0xffffffffu, (*abort && any_mma) ? 1 : 0, 0) != 0;
      if (drain && elect_one()) {
        // Drain the MMAs already issued before TMEM is released.
        const volatile int no_abort = 0;
        tc_commit_pair(map_to_rank(bar_drain, 0));
        mbar_wait_bounded(bar_drain, 0, &no_abort, 100000000ull);
      }
      __syncwarp();
    }
  } else {
    // -------------------------------------------------- epilogue --------
    const int quad = warp & 3;  // warps 2,3,4,5 -> TMEM lanes 64,96,0,32
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t acc_free_leader = map_to_rank(bar_acc_free, 0);
    const float alpha_a = __ldg(p.a_global);
    // alpha_A * alpha_B of the segment holding column `col` (segments are
    // whole 64-column epilogue subtiles)
    auto segment_scale = [&](int col) {
      int sg = 0;
      while (sg + 1 < p.nseg && col >= p.seg_end[sg]) ++sg;
      return __fmul_rn(alpha_a, __ldg(p.b_global + sg));
    };
    // NVFP4 output: the block step's constants and (d, r) table for the
    // output alpha, in the staging area (which the NVFP4 output does not use)
    BlockConsts qk;
    ScaleEntry* q_dr = reinterpret_cast<ScaleEntry*>(smem + OFF_STG);
    bool q_ok = true;
    if (EPI > 0) {
      const float qa = __ldg(p.q_alpha);
      q_ok = qa > 0.0f && !isinf(qa);  // a positive finite number, else nothing is written
      make_block_consts(q_ok ? qa : 1.0f, qk);
      fill_scale_table(q_ok ? qa : 1.0f, q_dr, threadIdx.x - 64);  // 128 epilogue threads, 128 entries
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!q_ok && threadIdx.x == 64 && rank == 0 && pair == 0) p.ws->status = NVFP4_ERR_INVALID_ARG;
    }
    const int64_t q_rows_padded = (static_cast<int64_t>(p.M) + 127) / 128 * 128;
    // this warp's two staging buffers; lane 0 issues (and waits for) every
    // TMA store of the warp, so the bulk groups it waits on are its own
    const uint32_t stg0 = sbase + OFF_STG + static_cast<uint32_t>(quad) * 2 * STG_BYTES;
    const uint64_t pol_stream = l2_policy_evict_first();  // Y is written once: do not let it evict B
    uint32_t nstore = 0;
    uint32_t local = 0;
    for (uint32_t tile = pair; tile < p.num_tiles; tile += npairs, ++local) {
      bool ok = mbar_wait_bounded(bar_acc_full, local & 1u, abort, p.timeout_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        if (lane == 0 && !*abort) record_timeout(p, abort, 3);
        break;
      }
      tc_fence_after();
      int m0, n0;
      tile_origin(p, tile, m0, n0);
      const int row0 = m0 + static_cast<int>(rank) * HALF + quad * 32;  // this warp's first row
      const int row = row0 + lane;
      const bool odd = (local & 1u) != 0;
      const uint32_t acc = tmem + lane_base + (odd ? TM_ACC1 : 0u);
      // Buffer 0 is drained from its last subtile, buffer 1 from its first:
      // either way the shared columns 192..255 go first and are released
      // before anything is stored.
      for (int si = 0; si < 4; ++si) {
        const int sub = odd ? si : (si == 0 ? 3 : si - 1);
        uint32_t r[64];
        tmem_ld32(acc + sub * EPI_N, r);
        tmem_ld32(acc + sub * EPI_N + 32, r + 32);
        tmem_wait_ld();
        if (si == 0) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(acc_free_leader);
        }
        const int col0 = n0 + sub * static_cast<int>(EPI_N);
        if (EPI > 0) {
          // Y rounded to bf16 as the plain output would be, then the block
          // step over its four 16-column blocks (N % 64 == 0)
          if (col0 >= p.N || row >= q_rows_padded || !q_ok) continue;
          const float ab = segment_scale(col0);
          uint32_t scales4 = 0;
          uint32_t cw[8];
          if (row < p.M) {
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16x2(__uint_as_float(r[16 * blk + 2 * i]) * ab,
                                   __uint_as_float(r[16 * blk + 2 * i + 1]) * ab);
              uint2 codes;
              uint32_t scale;
              const uint4 lo = make_uint4(w[0], w[1], w[2], w[3]), hi = make_uint4(w[4], w[5], w[6], w[7]);
              uint32_t bmax;
              if (EPI == 1) bmax = quantize_block<false, kRuleMax>(lo, hi, qk, q_dr, codes, scale);
              else if (EPI == 2) bmax = quantize_block<true, kRuleMax>(lo, hi, qk, q_dr, codes, scale);
              else if (EPI == 3) bmax = quantize_block<true, kRuleMae>(lo, hi, qk, q_dr, codes, scale);
              else bmax = quantize_block<true, kRuleMse>(lo, hi, qk, q_dr, codes, scale);
              if (bmax >= 0x7F80u) {  // Inf/NaN in the block: written as zeros, reported
                codes = make_uint2(0u, 0u);
                scale = 0u;
                p.ws->status = NVFP4_ERR_NONFINITE;
              }
              cw[2 * blk] = codes.x;
              cw[2 * blk + 1] = codes.y;
              scales4 |= scale << (8 * blk);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.q_codes + static_cast<int64_t>(row) * (p.N / 2) + col0 / 2);
            dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          }
          const int64_t atom = (static_cast<int64_t>(row) >> 7) * (p.N / 64) + col0 / 64;
          *reinterpret_cast<uint32_t*>(p.q_scales + atom * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4) = scales4;
          continue;
        }
        if (row0 >= p.M || col0 >= p.N) continue;  // warp-uniform
        const float ab = segment_scale(col0);
        if (p.tma_store) {
          if (p.out_fp32) {
            // 64 fp32 columns = two 32-column boxes, one per staging buffer
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t buf = stg0 + h * STG_BYTES + lane * 128;
#pragma unroll
              for (int c = 0; c < 8; ++c) {
                const int i = h * 32 + c * 4;
                st_shared_v4(buf + ((c ^ (lane & 7)) << 4),
                             __float_as_uint(__uint_as_float(r[i]) * ab),
                             __float_as_uint(__uint_as_float(r[i + 1]) * ab),
                             __float_as_uint(__uint_as_float(r[i + 2]) * ab),
                             __float_as_uint(__uint_as_float(r[i + 3]) * ab));
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d_hint(&tmY, stg0, col0, row0, pol_stream);
              tma_store_2d_hint(&tmY, stg0 + STG_BYTES, col0 + 32, row0, pol_stream);
              bulk_commit_group();
            }
          } else {
            const uint32_t stg = stg0 + (nstore & 1u) * STG_BYTES;
            if (lane == 0) bulk_wait_group_read<1>();  // the store that used this buffer is done reading
            __syncwarp();
            const uint32_t buf = stg + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int i = c * 8;
              st_shared_v4(buf + ((c ^ (lane & 7)) << 4),
                           pack_bf16x2(__uint_as_float(r[i]) * ab, __uint_as_float(r[i + 1]) * ab),
                           pack_bf16x2(__uint_as_float(r[i + 2]) * ab, __uint_as_float(r[i + 3]) * ab),
                           pack_bf16x2(__uint_as_float(r[i + 4]) * ab, __uint_as_float(r[i + 5]) * ab),
                           pack_bf16x2(__uint_as_float(r[i + 6]) * ab, __uint_as_float(r[i + 7]) * ab));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d_hint(&tmY, stg, col0, row0, pol_stream);
              bulk_commit_group();
            }
            ++nstore;
          }
          continue;
        }
        // direct stores (Y not 16-byte aligned or pitched): one row per lane
        if (row >= p.M) continue;
        const bool full = p.vec_store && col0 + static_cast<int>(EPI_N) <= p.N;
        if (p.out_fp32) {
          float* dst = static_cast<float*>(p.y) + static_cast<int64_t>(row) * p.ldy + col0;
          if (full) {
#pragma unroll
            for (int i = 0; i < 64; i += 4)
              *reinterpret_cast<float4*>(dst + i) =
                  make_float4(__uint_as_float(r[i]) * ab, __uint_as_float(r[i + 1]) * ab,
                              __uint_as_float(r[i + 2]) * ab, __uint_as_float(r[i + 3]) * ab);
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (col0 + i < p.N) dst[i] = __uint_as_float(r[i]) * ab;
          }
        } else {
          __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.y) + static_cast<int64_t>(row) * p.ldy + col0;
          if (full) {
#pragma unroll
            for (int i = 0; i < 64; i += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(r[i]) * ab, __uint_as_float(r[i + 1]) * ab);
              v.y = pack_bf16x2(__uint_as_float(r[i + 2]) * ab, __uint_as_float(r[i + 3]) * ab);
              v.z = pack_bf16x2(__uint_as_float(r[i + 4]) * ab, __uint_as_float(r[i + 5]) * ab);
              v.w = pack_bf16x2(__uint_as_float(r[i + 6]) * ab, __uint_as_float(r[i + 7]) * ab);
              *reinterpret_cast<uint4*>(dst + i) = v;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i)
              if (col0 + i < p.N) dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]) * ab);
          }
        }
      }
    }
    // the staging buffers must not be released (CTA exit) while a TMA store
    // still reads them
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }

  tc_fence_before();
  cluster_sync_all();  // no CTA leaves while its pair may still touch its barriers or TMEM
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------ host --

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2D uint8 tensor map over a K-major code matrix [rows, K/2]: 128-byte x
// 128-row boxes with the 128-byte swizzle.
nvfp4_status make_code_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK_BYTES), static_cast<cuuint32_t>(HALF)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(codes) failed (%d)", (int)r);
  return NVFP4_OK;
}

// 3D uint32 tensor map over a swizzled scale buffer seen as
// [row blocks][K groups][128 words]: one 512-byte atom per (row block, K
// group); boxes of 4 K groups x `blocks` row blocks, zero-filled past the end.
// 2D tensor map over Y [M, N] (row pitch ldy elements) for the epilogue's TMA
// stores: boxes of 128 bytes x 32 rows with the 128-byte swizzle.
nvfp4_status make_output_map(CUtensorMap* map, void* y, int64_t M, int64_t N, int64_t ldy, bool fp32) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  const cuuint64_t esize = fp32 ? 4 : 2;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldy) * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 32};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(Y) failed (%d)", (int)r);
  return NVFP4_OK;
}

nvfp4_status make_scale_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K,
                            uint32_t blocks) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  const int64_t kgroups = K / 64, rblocks = (rows + 127) / 128;
  const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(kgroups), static_cast<cuuint64_t>(rblocks)};
  const cuuint64_t strides[2] = {512, static_cast<cuuint64_t>(512 * kgroups)};
  const cuuint32_t box[3] = {128, 4, blocks};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(NVFP4_ERR_CUDA, "cuTensorMapEncodeTiled(scales) failed (%d)", (int)r);
  return NVFP4_OK;
}

}  // namespace

// Test hooks (not part of the public header): bounded-wait timeout and
// debug flags for the next nvfp4_gemm calls on this process.
static uint64_t g_timeout_ns = 4000000000ull;  // 4 s
static int g_debug_flags = 0;

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

void nvfp4_testing_set_gemm_wait(uint64_t timeout_ns, int debug_flags) {
  g_timeout_ns = timeout_ns ? timeout_ns : 4000000000ull;
  g_debug_flags = debug_flags;
}

}  // extern "C"

namespace {

template <int EPI>
cudaError_t launch_gemm(int dev, unsigned grid, cudaStream_t s, bool pdl, const CUtensorMap& ta,
                        const CUtensorMap& tb, const CUtensorMap& tsa, const CUtensorMap& tsb,
                        const CUtensorMap& ty, const GemmParams& p) {
  // the shared-memory opt-in is an attribute of the kernel in this context
  static PerContextCache<int> attr;
  int done = 0;
  const cudaError_t attr_err = per_context(attr, dev, [](int* v) {
    *v = 1;
    return cudaFuncSetAttribute(gemm_kernel<EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(SMEM_BYTES));
  }, &done);
  if (attr_err != cudaSuccess) return attr_err;
  return launch_kernel(gemm_kernel<EPI>, dim3(grid), dim3(kThreads), SMEM_BYTES, s, pdl, ta, tb, tsa, tsb, ty, p);
}

// A GEMM checked and ready to launch: tensor maps and kernel parameters.
struct GemmLaunch {
  CUtensorMap ta, tb, tsa, tsb, ty;
  GemmParams p;
  unsigned grid;
  int epi;
  int dev;
  void* workspace;
};

// Checks the arguments and prepares the launch; enqueues nothing.
// epi: 0 = bf16 / fp32 Y; 1..4 = NVFP4 Y (q_* arguments), see gemm_kernel.
nvfp4_status gemm_prepare(GemmLaunch* L, const char* fn, const void* a_codes, const void* a_scales,
                          const float* a_global, const void* b_codes, const void* b_scales,
                          const float* b_global, const int64_t* seg_ends, int nseg, int64_t M, int64_t N,
                          int64_t K, void* y, int64_t ldy, int out_dtype, void* workspace,
                          size_t workspace_bytes, int epi, const float* q_alpha, void* q_codes,
                          void* q_scales) {
  if (!a_codes || !a_scales || !a_global || !b_codes || !b_scales || !b_global || !y || !workspace)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  if (epi > 0) {
    if (!q_alpha || !q_codes || !q_scales) return set_error(NVFP4_ERR_INVALID_ARG, "%s: null pointer argument", fn);
    if (N % 64 != 0) return set_error(NVFP4_ERR_INVALID_ARG, "%s: need N %% 64 == 0 for an NVFP4 output", fn);
    if (!aligned16(q_codes) || !aligned16(q_scales) || (reinterpret_cast<uintptr_t>(q_alpha) & 3u))
      return set_error(NVFP4_ERR_INVALID_ARG, "%s: misaligned buffer", fn);
  }
  if (M < 1 || N < 1 || K < 64 || K % 64 != 0)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: need M, N >= 1 and K a positive multiple of 64 (M=%lld N=%lld K=%lld)", fn,
                     (long long)M, (long long)N, (long long)K);
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: dimension too large", fn);
  if (ldy < N || ldy > (int64_t{1} << 40)) return set_error(NVFP4_ERR_INVALID_ARG, "%s: need N <= ldy <= 2^40", fn);
  if (out_dtype != NVFP4_OUT_BF16 && out_dtype != NVFP4_OUT_FP32)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: unknown out_dtype %d", fn, out_dtype);
  if (!aligned16(a_codes) || !aligned16(b_codes) || !aligned16(a_scales) || !aligned16(b_scales) ||
      (reinterpret_cast<uintptr_t>(y) & (out_dtype == NVFP4_OUT_FP32 ? 3u : 1u)) ||
      !aligned16(workspace) ||
      (reinterpret_cast<uintptr_t>(a_global) & 3u) ||
      (reinterpret_cast<uintptr_t>(b_global) & 3u))
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: misaligned buffer", fn);
  if (nseg < 1 || nseg > kMaxSegments)
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: need 1 <= nseg <= %d", fn, kMaxSegments);
  for (int i = 0; i < nseg; ++i) {
    const int64_t lo = i ? seg_ends[i - 1] : 0;
    if (seg_ends[i] <= lo || (i + 1 < nseg ? seg_ends[i] % 64 != 0 : seg_ends[i] != N))
      return set_error(NVFP4_ERR_INVALID_ARG,
                       "%s: segment ends must ascend, be multiples of 64, and end at N", fn);
  }
  if (workspace_bytes < nvfp4_gemm_workspace_bytes())
    return set_error(NVFP4_ERR_INVALID_ARG, "%s: workspace too small", fn);
  int dev = 0, sms = 0;
  nvfp4_status st = check_device(&dev, &sms);
  if (st != NVFP4_OK) return st;

  if ((st = make_code_map(&L->ta, a_codes, M, K)) != NVFP4_OK) return st;
  if ((st = make_code_map(&L->tb, b_codes, N, K)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&L->tsa, a_scales, M, K, 1)) != NVFP4_OK) return st;
  if ((st = make_scale_map(&L->tsb, b_scales, N, K, 2)) != NVFP4_OK) return st;

  GemmParams& p = L->p;
  p.a_global = a_global;
  p.b_global = b_global;
  p.nseg = nseg;
  for (int i = 0; i < kMaxSegments; ++i) p.seg_end[i] = static_cast<int>(i < nseg ? seg_ends[i] : N);
  p.y = y;
  p.ws = static_cast<WorkspaceHeader*>(workspace);
  p.ldy = ldy;
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.kgroups = static_cast<uint32_t>(K / 64);
  p.ktiles = static_cast<uint32_t>((K + 255) / 256);
  p.n_tiles = static_cast<uint32_t>((N + BN - 1) / BN);
  p.m_tiles = static_cast<uint32_t>((M + BM - 1) / BM);
  const int64_t num_tiles = ((M + BM - 1) / BM) * static_cast<int64_t>(p.n_tiles);
  if (num_tiles > 0x7FFFFFFFll) return set_error(NVFP4_ERR_INVALID_ARG, "%s: too many tiles", fn);
  p.num_tiles = static_cast<uint32_t>(num_tiles);
  p.out_fp32 = out_dtype == NVFP4_OUT_FP32;
  p.vec_store = aligned16(y) && ((ldy * (p.out_fp32 ? 4 : 2)) % 16 == 0);
  p.tma_store = p.vec_store && epi == 0;
  p.q_alpha = q_alpha;
  p.q_codes = static_cast<uint8_t*>(q_codes);
  p.q_scales = static_cast<uint8_t*>(q_scales);
  std::memset(&L->ty, 0, sizeof(L->ty));
  if (p.tma_store && (st = make_output_map(&L->ty, y, M, N, ldy, p.out_fp32 != 0)) != NVFP4_OK) return st;
  p.timeout_ns = g_timeout_ns;
  p.debug_flags = g_debug_flags;
  // one CTA pair per two SMs, never more pairs than tiles
  const int64_t pairs = std::max<int64_t>(1, std::min<int64_t>(num_tiles, sms / 2));
  L->grid = static_cast<unsigned>(2 * pairs);
  L->epi = epi;
  L->dev = dev;
  L->workspace = workspace;
  return NVFP4_OK;
}

// Enqueues the status-word reset (unless the caller already did) and the
// kernel, as a programmatic dependent of the previous kernel when `pdl` is
// set (only useful when that kernel immediately precedes it on the stream).
nvfp4_status gemm_enqueue(const GemmLaunch& L, cudaStream_t s, bool clear_status, bool pdl) {
  cudaError_t e;
  if (clear_status && (e = cudaMemsetAsync(L.workspace, 0, sizeof(WorkspaceHeader), s)) != cudaSuccess)
    return cuda_status(e, "cudaMemsetAsync(status)");
  switch (L.epi) {
    case 0: e = launch_gemm<0>(L.dev, L.grid, s, pdl, L.ta, L.tb, L.tsa, L.tsb, L.ty, L.p); break;
    case 1: e = launch_gemm<1>(L.dev, L.grid, s, pdl, L.ta, L.tb, L.tsa, L.tsb, L.ty, L.p); break;
    case 2: e = launch_gemm<2>(L.dev, L.grid, s, pdl, L.ta, L.tb, L.tsa, L.tsb, L.ty, L.p); break;
    case 3: e = launch_gemm<3>(L.dev, L.grid, s, pdl, L.ta, L.tb, L.tsa, L.tsb, L.ty, L.p); break;
    default: e = launch_gemm<4>(L.dev, L.grid, s, pdl, L.ta, L.tb, L.tsa, L.tsb, L.ty, L.p); break;
  }
  if (e != cudaSuccess) return cuda_status(e, "gemm_kernel launch");
  return NVFP4_OK;
}

nvfp4_status gemm_impl(const char* fn, const void* a_codes, const void* a_scales, const float* a_global,
                       const void* b_codes, const void* b_scales, const float* b_global,
                       const int64_t* seg_ends, int nseg, int64_t M, int64_t N, int64_t K, void* y,
                       int64_t ldy, int out_dtype, void* workspace, size_t workspace_bytes,
                       void* stream, int epi = 0, const float* q_alpha = nullptr,
                       void* q_codes = nullptr, void* q_scales = nullptr) {
  GemmLaunch L;
  nvfp4_status st = gemm_prepare(&L, fn, a_codes, a_scales, a_global, b_codes, b_scales, b_global, seg_ends,
                                 nseg, M, N, K, y, ldy, out_dtype, workspace, workspace_bytes, epi, q_alpha,
                                 q_codes, q_scales);
  if (st != NVFP4_OK) return st;
  return gemm_enqueue(L, static_cast<cudaStream_t>(stream), true, false);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_gemm(const void* a_codes, const void* a_scales, const float* a_global,
                        const void* b_codes, const void* b_scales, const float* b_global,
                        int64_t M, int64_t N, int64_t K, void* y, int64_t ldy, int out_dtype,
                        void* workspace, size_t workspace_bytes, void* stream) {
  const int64_t end = N;
  return gemm_impl("nvfp4_gemm", a_codes, a_scales, a_global, b_codes, b_scales, b_global, &end, 1,
                   M, N, K, y, ldy, out_dtype, workspace, workspace_bytes, stream);
}

nvfp4_status nvfp4_gemm_quantized(const void* a_codes, const void* a_scales, const float* a_global,
                                  const void* b_codes, const void* b_scales, const float* b_global,
                                  int64_t M, int64_t N, int64_t K, int mode, int rule, const float* y_alpha,
                                  void* y_codes, void* y_scales, void* workspace, size_t workspace_bytes,
                                  void* stream) {
  if (mode != NVFP4_MODE_SIX && mode != NVFP4_MODE_FOUR_OVER_SIX)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_gemm_quantized: unknown mode %d", mode);
  if (rule != NVFP4_RULE_MAX && rule != NVFP4_RULE_MAE && rule != NVFP4_RULE_MSE)
    return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_gemm_quantized: unknown rule %d", rule);
  const int epi = mode == NVFP4_MODE_SIX ? 1 : (rule == NVFP4_RULE_MAX ? 2 : rule == NVFP4_RULE_MAE ? 3 : 4);
  const int64_t end = N;
  // y / ldy are not written with an NVFP4 output; y_codes stands in for the pointer checks
  return gemm_impl("nvfp4_gemm_quantized", a_codes, a_scales, a_global, b_codes, b_scales, b_global, &end,
                   1, M, N, K, y_codes, N, NVFP4_OUT_BF16, workspace, workspace_bytes, stream, epi, y_alpha,
                   y_codes, y_scales);
}

nvfp4_status nvfp4_quantize_gemm(const void* x, int64_t M, int64_t K, int64_t ldx, int mode, int rule,
                                 float fp8_max, void* x_codes, void* x_scales, float* x_global_scale,
                                 void* x_workspace, size_t x_workspace_bytes, const void* w_codes,
                                 const void* w_scales, const float* w_global, int64_t N, void* y, int64_t ldy,
                                 int out_dtype, void* workspace, size_t workspace_bytes, void* stream) {
  const char* fn = "nvfp4_quantize_gemm";
  // every check of both halves before anything is enqueued
  nvfp4_status st = quantize_rows_check(fn, x, M, K, ldx, mode, rule, fp8_max, x_codes, x_scales,
                                        x_global_scale, x_workspace, x_workspace_bytes);
  if (st != NVFP4_OK) return st;
  GemmLaunch L;
  const int64_t end = N;
  if ((st = gemm_prepare(&L, fn, x_codes, x_scales, x_global_scale, w_codes, w_scales, w_global, &end, 1, M, N, K,
                         y, ldy, out_dtype, workspace, workspace_bytes, 0, nullptr, nullptr, nullptr)) != NVFP4_OK)
    return st;
  // The GEMM's status word is cleared first, so that on the stream the GEMM
  // follows the quantize kernel directly and starts as its programmatic
  // dependent: its prologue overlaps the quantizer's tail.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(WorkspaceHeader), s);
  if (e != cudaSuccess) return cuda_status(e, "cudaMemsetAsync(status)");
  if ((st = quantize_rows_enqueue(fn, x, M, K, ldx, mode, rule, fp8_max, x_codes, x_scales, x_global_scale,
                                  x_workspace, x_workspace_bytes, stream)) != NVFP4_OK)
    return st;
  return gemm_enqueue(L, s, false, true);
}

}  // extern "C"

namespace {

// The augmented-channel layer in one call (with the activations' RMSNorm
// fused ahead when gamma is non-null).
nvfp4_status arc_gemm_impl(const char* fn, const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                           float eps, const int32_t* perm, int64_t S, int mode, int rule, float fp8_max,
                           void* x_codes, void* x_scales, float* x_global_scale, void* x_workspace,
                           size_t x_workspace_bytes, const void* w_codes, const void* w_scales,
                           const float* w_global, int64_t N, void* y, int64_t ldy, int out_dtype, void* workspace,
                           size_t workspace_bytes, void* stream) {
  nvfp4_status st = quantize_arc_check(fn, x, M, K, ldx, perm, S, 0, mode, rule, fp8_max, x_codes, x_scales,
                                       x_global_scale, x_workspace, x_workspace_bytes, gamma, eps);
  if (st != NVFP4_OK) return st;
  GemmLaunch L;
  const int64_t end = N;
  if ((st = gemm_prepare(&L, fn, x_codes, x_scales, x_global_scale, w_codes, w_scales, w_global, &end, 1, M, N,
                         K + S, y, ldy, out_dtype, workspace, workspace_bytes, 0, nullptr, nullptr, nullptr)) !=
      NVFP4_OK)
    return st;
  // as in nvfp4_quantize_gemm: the status reset first, then the quantizer's
  // kernels and the GEMM back to back, each a programmatic dependent
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(WorkspaceHeader), s);
  if (e != cudaSuccess) return cuda_status(e, "cudaMemsetAsync(status)");
  if ((st = quantize_arc_enqueue(fn, x, M, K, ldx, perm, S, 0, mode, rule, fp8_max, x_codes, x_scales,
                                 x_global_scale, x_workspace, x_workspace_bytes, stream, gamma, eps)) != NVFP4_OK)
    return st;
  return gemm_enqueue(L, s, false, true);
}

}  // namespace

extern "C" {

nvfp4_status nvfp4_quantize_arc_gemm(const void* x, int64_t M, int64_t K, int64_t ldx, const int32_t* perm,
                                     int64_t S, int mode, int rule, float fp8_max, void* x_codes, void* x_scales,
                                     float* x_global_scale, void* x_workspace, size_t x_workspace_bytes,
                                     const void* w_codes, const void* w_scales, const float* w_global, int64_t N,
                                     void* y, int64_t ldy, int out_dtype, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  return arc_gemm_impl("nvfp4_quantize_arc_gemm", x, M, K, ldx, nullptr, 0.0f, perm, S, mode, rule, fp8_max,
                       x_codes, x_scales, x_global_scale, x_workspace, x_workspace_bytes, w_codes, w_scales,
                       w_global, N, y, ldy, out_dtype, workspace, workspace_bytes, stream);
}

nvfp4_status nvfp4_quantize_arc_rmsnorm_gemm(const void* x, int64_t M, int64_t K, int64_t ldx, const void* gamma,
                                             float eps, const int32_t* perm, int64_t S, int mode, int rule,
                                             float fp8_max, void* x_codes, void* x_scales, float* x_global_scale,
                                             void* x_workspace, size_t x_workspace_bytes, const void* w_codes,
                                             const void* w_scales, const float* w_global, int64_t N, void* y,
                                             int64_t ldy, int out_dtype, void* workspace, size_t workspace_bytes,
                                             void* stream) {
  const char* fn = "nvfp4_quantize_arc_rmsnorm_gemm";
  if (!gamma) return set_error(NVFP4_ERR_INVALID_ARG, "%s: null pointer argument", fn);
  return arc_gemm_impl(fn, x, M, K, ldx, gamma, eps, perm, S, mode, rule, fp8_max, x_codes, x_scales,
                       x_global_scale, x_workspace, x_workspace_bytes, w_codes, w_scales, w_global, N, y, ldy,
                       out_dtype, workspace, workspace_bytes, stream);
}

nvfp4_status nvfp4_gemm_segmented(const void* a_codes, const void* a_scales, const float* a_global,
                                  const void* b_codes, const void* b_scales, const float* b_globals,
                                  const int64_t* seg_ends, int nseg, int64_t M, int64_t N, int64_t K,
                                  void* y, int64_t ldy, int out_dtype, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  if (!seg_ends) return set_error(NVFP4_ERR_INVALID_ARG, "nvfp4_gemm_segmented: null seg_ends");
  return gemm_impl("nvfp4_gemm_segmented", a_codes, a_scales, a_global, b_codes, b_scales, b_globals,
                   seg_ends, nseg, M, N, K, y, ldy, out_dtype, workspace, workspace_bytes, stream);
}

}  // extern "C"
