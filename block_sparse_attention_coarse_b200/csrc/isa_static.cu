// isa_forward_static: the ISA forward (planning + attention) for callers that
// cannot allocate device memory.  Some callers cannot give the library a
// workspace: code running where cudaMalloc is not allowed or not wanted
// (inside a custom allocator or memory-pool callback, a host function that
// must not allocate, or a tight real-time loop that forbids allocation) and
// bindings that have no device allocator of their own.  This entry point keeps
// the plan in a fixed device array that is part of the library image, so the
// caller only passes its inputs and output.
//
// The array has a fixed maximum size, kStaticScratchBytes; problems whose plan
// needs more are rejected with ISA_ERR_WORKSPACE before anything is launched.
// Every GPU that loads the library holds the array until the process exits.
//
// All calls share the one array and it keeps the last call's contents.  The
// planning kernels rewrite every plan entry they read back and isa_plan clears
// the device status word, so no other clearing is needed.  Calls that overlap
// on the GPU (different streams without ordering between them, or several host
// threads) race on the array: order them.  isa_forward_static_status copies
// the array's status word out, so that a caller can see a device wait that
// ran out.
//
// The first call on a device looks the array up (cudaGetSymbolAddress) and
// may make the driver load the library's device code, the array included:
// make it where allocation is allowed, as a warm-up.  The cached address
// belongs to the device's context as it was then; after cudaDeviceReset it is
// stale and this entry point must not be used on that device again.
#include <cstdio>
#include <mutex>

#include "isa_common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
constexpr int kMaxDevices = 64;

// In host code this name is only a stand-in for the device array; its device
// address comes from cudaGetSymbolAddress, per device.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mu;
void* g_static_ptr[kMaxDevices] = {};
// device address of the status word inside the array, per device (set by
// the first call on that device)
const int32_t* g_static_status[kMaxDevices] = {};

}  // namespace

extern "C" isa_status isa_forward_static(const isa_params* p, const void* q, const void* k, const void* v, void* out,
                                         float* lse, void* stream) {
  size_t need = 0;
  isa_status s = isa_plan_workspace_size(p, &need);
  if (s != ISA_OK) return s;
  char msg[200];
  if (need > kStaticScratchBytes) {
    snprintf(msg, sizeof(msg), "isa_forward_static: the plan needs %zu bytes, more than the %zu-byte fixed device array",
             need, kStaticScratchBytes);
    isa::set_last_error(msg);
    return ISA_ERR_WORKSPACE;
  }
  if (!q) {
    isa::set_last_error("q is NULL");
    return ISA_ERR_INVALID_ARG;
  }
  if ((s = isa::bind_device_of(q, "q")) != ISA_OK) return s;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "isa_forward_static: no usable current device (%s)", cudaGetErrorString(e));
    isa::set_last_error(msg);
    return ISA_ERR_CUDA;
  }
  void* ptr = nullptr;
  {
    // first call on a device: look up the device address of the array
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_ptr[dev]) {
      e = cudaGetSymbolAddress(&g_static_ptr[dev], g_static_scratch);
      if (e != cudaSuccess) {
        g_static_ptr[dev] = nullptr;
        snprintf(msg, sizeof(msg), "isa_forward_static: cudaGetSymbolAddress failed (%s)", cudaGetErrorString(e));
        isa::set_last_error(msg);
        return ISA_ERR_CUDA;
      }
    }
    ptr = g_static_ptr[dev];
    if (!g_static_status[dev]) {
      isa_plan_view view;
      if ((s = isa_plan_view_get(p, ptr, kStaticScratchBytes, &view)) != ISA_OK) return s;
      g_static_status[dev] = view.status;
    }
  }
  s = isa_plan(p, q, k, v, ptr, kStaticScratchBytes, stream);
  if (s != ISA_OK) return s;
  return isa_forward(p, q, k, v, ptr, kStaticScratchBytes, out, lse, stream);
}

extern "C" isa_status isa_forward_static_status(int32_t device, int32_t* dst, void* stream) {
  char msg[200];
  if (!dst) {
    isa::set_last_error("isa_forward_static_status: dst is NULL");
    return ISA_ERR_INVALID_ARG;
  }
  if (device < 0 || device >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "isa_forward_static_status: device %d out of range", (int)device);
    isa::set_last_error(msg);
    return ISA_ERR_INVALID_ARG;
  }
  const int32_t* src = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    src = g_static_status[device];
  }
  if (!src) {
    snprintf(msg, sizeof(msg), "isa_forward_static_status: isa_forward_static has not run on device %d",
             (int)device);
    isa::set_last_error(msg);
    return ISA_ERR_INVALID_ARG;
  }
  cudaError_t e = cudaSetDevice(device);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(dst, src, sizeof(int32_t), cudaMemcpyDefault, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "isa_forward_static_status: copy failed (%s)", cudaGetErrorString(e));
    isa::set_last_error(msg);
    return ISA_ERR_CUDA;
  }
  return ISA_OK;
}
