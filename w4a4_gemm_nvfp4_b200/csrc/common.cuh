// common.cuh -- host plumbing and sm_100a PTX helpers shared by the NVFP4
// kernels of libnvfp4.so.  Nothing here is shared with the CPU oracle.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>
#include <utility>

#include "nvfp4.h"

namespace nvfp4 {

// ------------------------------------------------------------------ host --

// Records a message for nvfp4_last_error_message() and returns `st`.
nvfp4_status set_error(nvfp4_status st, const char* fmt, ...);
// Returns NVFP4_OK when the current device is compute capability 10.0.
nvfp4_status check_device(int* device, int* num_sms);
// Turns a cudaError_t into NVFP4_ERR_CUDA with its message.
nvfp4_status cuda_status(cudaError_t err, const char* what);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// nvfp4_quantize's argument checks alone (no device check; enqueues nothing), and its whole work
// (checks, amax pass, quantize kernel), with `fn` naming the entry point in
// error messages: for entry points that quantize and then go on.
nvfp4_status quantize_rows_check(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                                 int rule, float fp8_max, const void* codes, const void* scales,
                                 const float* global_scale, const void* workspace, size_t workspace_bytes);
nvfp4_status quantize_rows_enqueue(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx, int mode,
                                   int rule, float fp8_max, void* codes, void* scales, float* global_scale,
                                   void* workspace, size_t workspace_bytes, void* stream);
// The same pair for nvfp4_quantize_arc; with `gamma` non-null, for
// nvfp4_quantize_arc_rmsnorm (augment 0, RMSNorm with gains gamma and eps).
nvfp4_status quantize_arc_check(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx,
                                const int32_t* perm, int64_t S, int augment, int mode, int rule, float fp8_max,
                                const void* codes, const void* scales, const float* global_scale,
                                const void* workspace, size_t workspace_bytes, const void* gamma = nullptr,
                                float eps = 0.0f);
nvfp4_status quantize_arc_enqueue(const char* fn, const void* x, int64_t rows, int64_t K, int64_t ldx,
                                  const int32_t* perm, int64_t S, int augment, int mode, int rule, float fp8_max,
                                  void* codes, void* scales, float* global_scale, void* workspace,
                                  size_t workspace_bytes, void* stream, const void* gamma = nullptr,
                                  float eps = 0.0f);

// Launches `kernel` on `stream`, as a programmatic dependent of the previous
// kernel on the stream when `pdl` is set (the kernel must then call
// pdl_wait() before touching memory that kernel uses).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                          bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The driver's unique id of the CUDA context current on this thread (ids are
// never reused within a process, unlike context handles), or 0 when no
// context is current or the driver cannot be asked.
uint64_t current_context_id();

// A value computed once per CUDA context of each device: kernel attributes,
// occupancy and symbol addresses belong to the context that loaded the
// module, so a device whose primary context was reset (cudaDeviceReset) or
// replaced gets them computed again.
constexpr int kMaxDevices = 64;
template <typename T>
struct PerContextCache {
  std::mutex mu;
  uint64_t ctx[kMaxDevices] = {};
  T value[kMaxDevices] = {};
};
// The cached value for device `dev` (the current device) in the current
// context; `make(T*)` computes it (returning a cudaError_t) when the context
// changed or nothing is cached yet.  When no context id can be read the value
// is recomputed on every call.
template <typename T, typename Make>
cudaError_t per_context(PerContextCache<T>& c, int dev, Make make, T* out) {
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(c.mu);
  const uint64_t id = current_context_id();
  if (id == 0 || c.ctx[dev] != id) {
    T v{};
    const cudaError_t e = make(&v);
    if (e != cudaSuccess) return e;
    c.value[dev] = v;
    c.ctx[dev] = current_context_id();  // the computation may have created the context
  }
  *out = c.value[dev];
  return cudaSuccess;
}

// Status words live at the start of every workspace.
struct WorkspaceHeader {
  uint32_t status;      // nvfp4_status of the last kernel that used the workspace
  uint32_t detail;      // kernel-specific detail (e.g. which wait ran out)
  uint32_t pad[14];     // keeps the partials 64-byte aligned
};
static_assert(sizeof(WorkspaceHeader) == 64, "workspace header is 64 bytes");

// ---------------------------------------------------------------- device --

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// mbarrier primitives (shared::cta addresses)
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: spins on try_wait until the phase with `parity` completed,
// `*abort` became non-zero, or `timeout_ns` passed (on %globaltimer) since
// this wait first checked the clock.  The limit is on a lack of progress:
// every wait gets the whole timeout, however long the kernel has run.
// Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  const volatile int* abort,
                                                  uint64_t timeout_ns) {
  uint64_t start = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort) return false;
      const uint64_t now = global_timer_ns();
      if (start == 0) start = now;
      else if (now - start > timeout_ns) return false;
    }
  }
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "elect.sync _|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// TMA for one CTA of a CTA pair (cta_group::2): the destination is this CTA's
// shared memory, the mbarrier `bar_cluster` may live in either CTA of the pair
// (a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t c0, int32_t c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t c0, int32_t c1,
                                                 int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// L2 eviction-priority policies for the cache-hinted copies below.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
// tma_load_2d_pair / tma_load_3d_pair with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap* map,
                                                      uint32_t bar_cluster, int32_t c0, int32_t c1,
                                                      uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair_hint(uint32_t dst, const CUtensorMap* map,
                                                      uint32_t bar_cluster, int32_t c0, int32_t c1,
                                                      int32_t c2, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1), "r"(c2), "l"(policy)
      : "memory");
}
// tma_store_2d with an L2 cache policy.
__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, uint32_t src, int32_t c0,
                                                  int32_t c1, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group.L2::cache_hint [%0, {%2, %3}], [%1], %4;" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Waits until at most N of this thread's committed bulk groups still read
// shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Waits until all of this thread's committed bulk groups have completed.
__device__ __forceinline__ void bulk_wait_group_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------ clusters --

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared-memory offset in CTA `rank`.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive (count 1) on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

// Programmatic dependent launch.  A kernel launched as a programmatic
// dependent of the previous kernel on its stream may start while that kernel
// still runs; pdl_wait() blocks until the previous kernel has completed and
// its memory writes are visible, so it must come before the first access to
// anything the previous kernel touches.  For a kernel launched normally it
// returns at once.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets a programmatic dependent of this grid start once every CTA of this
// grid has called it (or exited); the dependent still waits in pdl_wait().
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------- tcgen05 ----

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Pair versions (cta_group::2): TMEM allocated in both CTAs of the pair at once.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Arrive on the mbarrier at shared::cluster address `bar_cluster` (either CTA
// of the pair) once every previously issued cta_group::2 tcgen05 op of this
// thread completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar_cluster) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar_cluster)
      : "memory");
}

}  // namespace nvfp4
