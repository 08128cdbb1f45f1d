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
void* g_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device (looked up once
// per device, with that device current).
mova_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOVA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, noalloc_scratch) != cudaSuccess || p == nullptr) return MOVA_ERR_CUDA;
    g_addr[dev] = p;
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
  if (T == 0) return MOVA_OK;
  const size_t need = mova_workspace_size(T, d, E, k, n);
  if (need == 0) return mova_value_routed(x, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v,
                                          nullptr, nullptr, nullptr, 0, stream);  // reports the size error
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
