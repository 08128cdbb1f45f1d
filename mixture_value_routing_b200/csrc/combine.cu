// Fixed-order gather-combine.
//
//   v[t, :] = sum over slot = 0..k-1 (ascending) of w[t*k + slot] * P[pos[t*k + slot], :]
//
// P holds SiLU(Wv[e] x[t]) per (token, slot) pair, in grouped order; this
// weights each token's k rows by their routing weights and sums them in
// ascending slot order in fp32, rounding once at the store.  The (T, n) result, n = heads x 128, is the GQA
// value tensor ("MoVA: routing the value vectors, and why the KV cache does
// not notice", section "Where the routing happens": the mixture is reshaped
// into 8 heads of 128 and is exactly what a GQA v_proj produces).
//
// HBM-bound: every thread moves 8 consecutive outputs (16-byte loads of bf16
// rows, 2 x 16 bytes of fp32 rows); P rows are read once (streaming loads).
#include "common.cuh"
#include "internal.h"

namespace mova {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ void load8_p(const float* p, float out[8]) { load8_stream(p, out); }
__device__ __forceinline__ void load8_p(const __nv_bfloat16* p, float out[8]) { load8_stream(p, out); }

__device__ __forceinline__ void store8(float* p, const float v[8]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float v[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// KS > 0: k == KS known at compile time -- all slots' positions, weights and
// P vectors are loaded before the first multiply-add, so each thread keeps
// KS independent 16-byte loads in flight.  KS == 0: any k, slot by slot.
template <typename PT, typename OT, int KS>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const PT* __restrict__ P, const int32_t* __restrict__ pos,
               const float* __restrict__ w32, int T, int k, int n, OT* __restrict__ v) {
  // The next call's plane split may start now: it touches nothing this
  // kernel reads, and waits for this grid before it ends.
  pdl_trigger();
  pdl_wait();  // the expert rows of this call are complete and visible
  const int per_tok = n / 8;
  const long long total = static_cast<long long>(T) * per_tok;
  for (long long i = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * kThreads) {
    const int t = static_cast<int>(i / per_tok);
    const int c = static_cast<int>(i % per_tok) * 8;
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    if constexpr (KS > 0) {
      int p[KS];
      float ws[KS];
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        p[s] = pos[static_cast<size_t>(t) * KS + s];
        ws[s] = w32[static_cast<size_t>(t) * KS + s];
      }
      float pv[KS][8];
#pragma unroll
      for (int s = 0; s < KS; ++s) load8_p(P + static_cast<size_t>(p[s]) * n + c, pv[s]);
#pragma unroll
      for (int s = 0; s < KS; ++s)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(ws[s], pv[s][q], acc[q]);
    } else {
      for (int s = 0; s < k; ++s) {
        const int p = pos[static_cast<size_t>(t) * k + s];
        const float ws = w32[static_cast<size_t>(t) * k + s];
        float pv[8];
        load8_p(P + static_cast<size_t>(p) * n + c, pv);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(ws, pv[q], acc[q]);
      }
    }
    store8(v + static_cast<size_t>(t) * n + c, acc);
  }
}

template <typename PT, typename OT>
cudaError_t launch_t(const void* P, const int32_t* pos, const float* w32, int T, int k, int n,
                     void* v, cudaStream_t stream) {
  const long long total = static_cast<long long>(T) * (n / 8);
  long long blocks = (total + kThreads - 1) / kThreads;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (k == 4)
    return launch_pdl(combine_kernel<PT, OT, 4>, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                      stream, static_cast<const PT*>(P), pos, w32, T, k, n, static_cast<OT*>(v));
  return launch_pdl(combine_kernel<PT, OT, 0>, dim3(static_cast<unsigned>(blocks)), dim3(kThreads), 0,
                    stream, static_cast<const PT*>(P), pos, w32, T, k, n, static_cast<OT*>(v));
}

}  // namespace

cudaError_t launch_combine(const void* P, bool p_bf16, const int32_t* pos, const float* w32, int T,
                           int k, int n, void* v, mova_dtype v_dt, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  if (p_bf16) {
    if (v_dt == MOVA_BF16) return launch_t<__nv_bfloat16, __nv_bfloat16>(P, pos, w32, T, k, n, v, stream);
    return launch_t<__nv_bfloat16, float>(P, pos, w32, T, k, n, v, stream);
  }
  if (v_dt == MOVA_BF16) return launch_t<float, __nv_bfloat16>(P, pos, w32, T, k, n, v, stream);
  return launch_t<float, float>(P, pos, w32, T, k, n, v, stream);
}

}  // namespace mova
