// qlinear_forward_fixed_scratch: the forward pass for callers that cannot allocate device memory.
//
// Some callers are not allowed to allocate: an inference runtime that plans every byte of device
// memory up front and treats an allocation during a forward as a bug, a plugin inside a host
// application that exposes no allocator to it, or a real-time loop that must not hit the
// allocator's locks or its possible implicit synchronisation.  qlinear_forward needs a workspace
// from its caller; this entry point instead uses one scratch array that lives in the library
// itself (a file-scope __device__ array, so every GPU that loads the library holds it until the
// process exits).  The caller still passes x, y and the optional fp32 y.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "qlinear.h"

// Defined in qlinear.cu: sets the thread-local message ql_last_error() returns.
ql_status ql_set_error(ql_status status, const char* message);

namespace {

constexpr size_t kFixedScratchBytes = size_t(8) << 20;  // 8 MiB per device

__device__ __align__(256) unsigned char g_fixed_scratch[kFixedScratchBytes];

// In host code `g_fixed_scratch` names a host-side stand-in, not device memory: its device
// address must be looked up with the device current.  The address is cached per device ordinal
// together with the context it belongs to, and looked up again when the current context is a
// different one (after cudaDeviceReset the module is loaded anew and the array may move).
constexpr int kMaxDevices = 64;
struct ScratchEntry {
  CUcontext ctx = nullptr;
  void* addr = nullptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

ql_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ql_set_error(QL_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return ql_set_error(QL_ERR_UNSUPPORTED, "device ordinal beyond the fixed-scratch table");
  CtxGetCurrentFn get_ctx = ctx_get_current();
  if (get_ctx == nullptr) return ql_set_error(QL_ERR_CUDA, "cuCtxGetCurrent unavailable");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  CUcontext ctx = nullptr;
  get_ctx(&ctx);
  ScratchEntry& e = g_scratch[dev];
  if (e.addr == nullptr || ctx == nullptr || e.ctx != ctx) {
    void* p = nullptr;
    const cudaError_t err = cudaGetSymbolAddress(&p, g_fixed_scratch);   // makes a context current
    if (err != cudaSuccess || p == nullptr)
      return ql_set_error(QL_ERR_CUDA, "cudaGetSymbolAddress of the fixed scratch array failed");
    get_ctx(&ctx);
    e.ctx = ctx;
    e.addr = p;
  }
  *out = e.addr;
  return QL_OK;
}

}  // namespace

extern "C" ql_status qlinear_forward_fixed_scratch(const ql_linear* layer, const void* x_bf16,
                                                   int64_t M, void* y_bf16, float* y_f32,
                                                   ql_stream_t stream) {
  if (layer == nullptr || M < 0)
    return ql_set_error(QL_ERR_INVALID_ARG, "null layer or negative M");
  if (M == 0) return QL_OK;
  size_t need = 0;
  ql_status st = qlinear_workspace_bytes(layer, M, &need);
  if (st != QL_OK) return st;
  if (need > kFixedScratchBytes)
    return ql_set_error(QL_ERR_WORKSPACE,
                        "qlinear_forward_fixed_scratch: this M needs more workspace than the "
                        "library's 8 MiB fixed scratch; use qlinear_forward with a caller buffer");
  void* scratch = nullptr;
  st = scratch_for_current_device(&scratch);
  if (st != QL_OK) return st;
  return qlinear_forward(layer, x_bf16, M, y_bf16, y_f32, scratch, kFixedScratchBytes, stream);
}
