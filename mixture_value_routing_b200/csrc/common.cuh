// Shared device helpers of the MoVA CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mova.h"

namespace mova {

// Layout of the status block at the start of every workspace.
struct StatusBlock {
  int32_t code;        // 0 or a mova_status set by a device-side check
  int32_t detail;      // first offending item
  int32_t num_active;  // experts with at least one routed pair (written by the grouping)
  int32_t work_next;   // reserved for dynamic tile scheduling
};

__device__ __forceinline__ void raise_status(StatusBlock* sb, int32_t code, int32_t detail) {
  if (atomicCAS(&sb->code, 0, code) == 0) sb->detail = detail;
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Eight consecutive elements as fp32 (one 16-byte load for bf16, two for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float out[8]) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float out[8]) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

// Streaming (read-once) variants for expert weights: bypass L1 allocation
// and mark the lines evict-first in L2.
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p), "l"(evict_first_policy()));
  return r;
}
__device__ __forceinline__ void load8_stream(const __nv_bfloat16* p, float out[8]) {
  uint4 u = ld_stream_u4(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8_stream(const float* p, float out[8]) {
  uint4 a = ld_stream_u4(p);
  uint4 b = ld_stream_u4(p + 4);
  out[0] = __uint_as_float(a.x); out[1] = __uint_as_float(a.y);
  out[2] = __uint_as_float(a.z); out[3] = __uint_as_float(a.w);
  out[4] = __uint_as_float(b.x); out[5] = __uint_as_float(b.y);
  out[6] = __uint_as_float(b.z); out[7] = __uint_as_float(b.w);
}

// Programmatic dependent launch: wait for the predecessor grid (no-op when
// the kernel was launched without the attribute), and let the successor
// start its launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Logistic function and SiLU in fp32 (IEEE expf and division).
__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }
__device__ __forceinline__ float siluf_(float h) { return h / (1.0f + expf(-h)); }
// SiLU with the fast exponential and division intrinsics (relative error
// ~1e-6): used where the result is rounded to bf16 anyway.
__device__ __forceinline__ float silu_fast(float h) { return __fdividef(h, 1.0f + __expf(-h)); }

}  // namespace mova
