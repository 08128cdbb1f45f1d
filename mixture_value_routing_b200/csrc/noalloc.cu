// mova_value_routed_noalloc: the full value path with no allocation at all.
//
// Some callers cannot allocate device memory at the point where they need
// the value projection: code running inside a stream capture that must not
// add allocation nodes, custom allocators and memory pools that own all of
// the device memory and forbid outside cudaMalloc calls, or plug-ins whose
// host framework gives them only the tensors they compute on.  For them this
// entry point takes its workspace from a fixed array compiled into the
// library (every GPU that loads the library holds it until the process
// exits) instead of a caller-provided buffer, and calls no cudaMalloc,
// cudaFree or other allocating routine.
//
// The kernels and their order are exactly those of mova_value_routed.
#include <cuda.h>

#include <cstdio>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace mova {
namespace {

constexpr size_t kNoallocScratchBytes = static_cast<size_t>(MOVA_NOALLOC_SCRATCH_BYTES);

// The shared workspace.  In host code `noalloc_scratch` only names a host-side
// stand-in for the symbol, never a device address: the kernels get the
// address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the context the address was looked up in (its process-unique
// id) and the address.  A device reset, or another context made current on
// the same device, loads the module again at another address; the id then
// differs and the address is looked up afresh.
unsigned long long g_ctx_id[kMaxDevices] = {0};
void* g_addr[kMaxDevices] = {nullptr};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

void* driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return p;
}

// Process-unique id of the current context (0 if none or unavailable).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = reinterpret_cast<CtxGetCurrentFn>(driver_fn("cuCtxGetCurrent"));
  static CtxGetIdFn get_id = reinterpret_cast<CtxGetIdFn>(driver_fn("cuCtxGetId"));
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array for the current device and context:
// looked up with that device current, then reused while the same context is
// current.  Without a context id the address is looked up on every call.
mova_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOVA_ERR_CUDA;
  const unsigned long long id = current_context_id();
  std::lock_guard<std::mutex> lock(g_mu);
  if (id == 0 || g_addr[dev] == nullptr || g_ctx_id[dev] != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || p == nullptr) return MOVA_ERR_CUDA;
    g_addr[dev] = p;
    // The lookup makes the device's primary context current if none was:
    // record the id of the context the address belongs to.
    g_ctx_id[dev] = current_context_id();
  }
  *out = g_addr[dev];
  return MOVA_OK;
}

}  // namespace
}  // namespace mova

extern "C" mova_status mova_value_routed_noalloc(const void* x, mova_dtype x_dt, const float* Wr,
                                                 const float* br, const void* Wv, mova_dtype wv_dt,
                                                 int T, int d, int E, int k, int n, float scale,
                                                 void* v, void* stream) {
  const size_t need = mova_workspace_size(T, d, E, k, n);
  // T == 0 and invalid sizes: mova_value_routed validates the arguments
  // exactly as for a caller-provided workspace (for T == 0 it returns
  // MOVA_OK after the checks, touching nothing).
  if (T == 0 || need == 0)
    return mova_value_routed(x, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v, nullptr, nullptr,
                             nullptr, 0, stream);
  if (need > mova::kNoallocScratchBytes) {
    fprintf(stderr,
            "mova_value_routed_noalloc: T=%d d=%d E=%d k=%d n=%d needs %zu bytes of workspace, "
            "more than the %zu-byte built-in scratch\n",
            T, d, E, k, n, need, mova::kNoallocScratchBytes);
    return MOVA_ERR_UNSUPPORTED;
  }
  void* ws = nullptr;
  const mova_status st = mova::scratch_for_current_device(&ws);
  if (st != MOVA_OK) return st;
  return mova_value_routed(x, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v, nullptr, nullptr, ws,
                           mova::kNoallocScratchBytes, stream);
}
