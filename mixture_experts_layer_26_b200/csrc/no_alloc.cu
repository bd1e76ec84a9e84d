// fused_moe_static_workspace: the one-call layer for callers that cannot allocate
// device memory.
//
// Some callers have no way to get device memory for the workspace: a plugin loaded
// into a serving process whose framework has already reserved the GPU's memory in its
// own pool and hands the plugin no allocator, or a latency-critical caller that must
// not call cudaMalloc / cudaFree because they can synchronise the device.  For them
// the workspace lives in a file-scope __device__ array of kStaticWsBytes that the
// library owns: every GPU that loads this library keeps that array until the process
// exits.  The caller still passes all inputs and the output.
//
// The array's name is a host-side stand-in in host code, not a device address, so the
// first call on each device, with that device current, asks the runtime for the
// array's device address (cudaGetSymbolAddress) and caches it; that first call should
// come before any stream capture.  Every call shares the one array and it keeps the
// last call's contents, so each call clears the workspace header (which holds the
// sticky device status word) before it runs; calls that overlap on the GPU (on
// different streams, or from different threads) race on the array and must be
// serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "fmoe_common.cuh"
#include "fused_moe.h"

namespace {

constexpr size_t kStaticWsBytes = FUSED_MOE_STATIC_WS_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

std::mutex g_mu;
void* g_ws_ptr[kMaxDevices] = {};

// Device address of g_static_ws on the current device (nullptr on failure).
void* static_ws_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ws_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || p == nullptr) return nullptr;
    g_ws_ptr[dev] = p;
  }
  return g_ws_ptr[dev];
}

}  // namespace

extern "C" fmoe_status fused_moe_static_workspace(const fmoe_dims* dims, const void* x,
                                                  const void* router_w, const void* w13,
                                                  const void* w2, const fmoe_scales* scales,
                                                  void* out, int32_t* device_status,
                                                  fmoe_stream stream) {
  const size_t need = fused_moe_workspace_size(dims);  // 0 for invalid dims
  if (need == 0) return FMOE_ERR_INVALID_ARG;
  if (dims->T == 0) return FMOE_OK;
  if (need > kStaticWsBytes) return FMOE_ERR_WORKSPACE;  // too large for the static array
  if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
    return FMOE_ERR_UNSUPPORTED;
  void* ws = static_ws_address();
  if (ws == nullptr) return FMOE_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the previous call's status word must not leak into this one
  if (cudaMemsetAsync(ws, 0, sizeof(fmoe::WsHeader), s) != cudaSuccess) return FMOE_ERR_CUDA;
  const fmoe_status st = fused_moe(dims, x, router_w, w13, w2, scales, out, ws, kStaticWsBytes, stream);
  if (st != FMOE_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return FMOE_ERR_CUDA;
  return FMOE_OK;
}
