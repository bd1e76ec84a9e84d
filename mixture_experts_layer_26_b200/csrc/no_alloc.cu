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
// Every argument check (the same ones fused_moe runs, then the size limit) comes
// before any CUDA call.  The array's name is a host-side stand-in in host code, not a
// device address, so every call asks the runtime for the array's device address on the
// current device (cudaGetSymbolAddress: a host-side lookup that enqueues nothing).
// Nothing is cached, so a call after cudaDeviceReset or under another context of the
// same device gets that context's address.  The first call in a context loads the
// library's module there, so make it before any stream capture.  Every call shares the
// one array and it keeps the last call's contents, so each call first clears the span
// fused_moe_workspace_init clears (the header with the sticky status word and the
// router's tile counters); calls that overlap on the GPU (on different streams, or from
// different threads) race on the array and must be serialised by the caller.
#include <cuda_runtime.h>

#include "fmoe_kernels.h"
#include "fused_moe.h"

namespace {

constexpr size_t kStaticWsBytes = FUSED_MOE_STATIC_WS_BYTES;

static __device__ __align__(256) unsigned char g_static_ws[kStaticWsBytes];

}  // namespace

extern "C" fmoe_status fused_moe_static_workspace(const fmoe_dims* dims, const void* x,
                                                  const void* router_w, const void* w13,
                                                  const void* w2, const fmoe_scales* scales,
                                                  void* out, int32_t* device_status,
                                                  fmoe_stream stream) {
  // argument checks first, with fused_moe's own status codes; no CUDA call before them
  const fmoe_status arg = fmoe::check_layer_args(dims, x, router_w, w13, w2, scales, out);
  if (arg != FMOE_OK) return arg;
  if (dims->T == 0) return FMOE_OK;
  if (device_status != nullptr && (reinterpret_cast<uintptr_t>(device_status) & 3u) != 0)
    return FMOE_ERR_UNSUPPORTED;
  if (fused_moe_workspace_size(dims) > kStaticWsBytes) return FMOE_ERR_WORKSPACE;

  void* ws = nullptr;
  if (cudaGetSymbolAddress(&ws, g_static_ws) != cudaSuccess || ws == nullptr) {
    (void)cudaGetLastError();
    return FMOE_ERR_CUDA;
  }
  // the previous call's status word and any router counter it left behind must not
  // leak into this one
  fmoe_status st = fused_moe_workspace_init(ws, kStaticWsBytes, stream);
  if (st != FMOE_OK) return st;
  st = fused_moe(dims, x, router_w, w13, w2, scales, out, ws, kStaticWsBytes, stream);
  if (st != FMOE_OK) return st;
  if (device_status != nullptr &&
      cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FMOE_ERR_CUDA;
  return FMOE_OK;
}
