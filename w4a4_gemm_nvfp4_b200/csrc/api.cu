// api.cu -- status plumbing, buffer-size helpers and the device-status read
// of the nvfp4 C ABI.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "common.cuh"

namespace nvfp4 {

static thread_local char g_msg[512] = "";

nvfp4_status set_error(nvfp4_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

nvfp4_status cuda_status(cudaError_t err, const char* what) {
  if (err == cudaSuccess) return NVFP4_OK;
  return set_error(NVFP4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err),
                   cudaGetErrorName(err));
}

// Driver entry points reached through the runtime (the library does not link
// libcuda): the current context and its process-unique id.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

uint64_t current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Per-device capability cache (compute capability and SM count).
static int g_dev_ok[kMaxDevices];      // 0 unknown, 1 sm_100, -1 other
static int g_dev_sms[kMaxDevices];
static std::mutex g_dev_mu;

nvfp4_status check_device(int* device, int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return set_error(NVFP4_ERR_UNSUPPORTED_DEVICE, "device %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_dev_ok[dev] == 0) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_status(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_status(e, "cudaDeviceGetAttribute");
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_status(e, "cudaDeviceGetAttribute");
    g_dev_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
    g_dev_sms[dev] = sms;
    if (g_dev_ok[dev] < 0)
      return set_error(NVFP4_ERR_UNSUPPORTED_DEVICE,
                       "device %d is compute capability %d.%d; this library is built for sm_100a",
                       dev, major, minor);
  }
  if (g_dev_ok[dev] < 0)
    return set_error(NVFP4_ERR_UNSUPPORTED_DEVICE, "device %d is not compute capability 10.0", dev);
  if (device) *device = dev;
  if (num_sms) *num_sms = g_dev_sms[dev];
  return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_codes_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * 128u * static_cast<size_t>(K / 16);
}

size_t nvfp4_gemm_workspace_bytes(void) { return sizeof(WorkspaceHeader); }

const char* nvfp4_status_string(nvfp4_status st) {
  switch (st) {
    case NVFP4_OK: return "NVFP4_OK";
    case NVFP4_ERR_INVALID_ARG: return "NVFP4_ERR_INVALID_ARG";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "NVFP4_ERR_UNSUPPORTED_DEVICE";
    case NVFP4_ERR_NONFINITE: return "NVFP4_ERR_NONFINITE";
    case NVFP4_ERR_TIMEOUT: return "NVFP4_ERR_TIMEOUT";
    case NVFP4_ERR_CUDA: return "NVFP4_ERR_CUDA";
  }
  return "NVFP4_ERR_UNKNOWN";
}

const char* nvfp4_last_error_message(void) { return g_msg; }

nvfp4_status nvfp4_get_device_status(const void* workspace, void* stream) {
  if (!workspace || !aligned16(workspace))
    return set_error(NVFP4_ERR_INVALID_ARG, "workspace must be a non-null 16-byte aligned pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e, "cudaStreamSynchronize");
  WorkspaceHeader h;
  e = cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e, "cudaMemcpy(status)");
  switch (h.status) {
    case NVFP4_OK: case NVFP4_ERR_INVALID_ARG: case NVFP4_ERR_NONFINITE: case NVFP4_ERR_TIMEOUT:
      return static_cast<nvfp4_status>(h.status);
    default:
      return set_error(NVFP4_ERR_CUDA, "workspace status word holds %u (never written?)", h.status);
  }
}

}  // extern "C"
