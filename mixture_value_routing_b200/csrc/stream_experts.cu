// Weight-streaming expert kernel for decode-sized batches (and the fp32 path).
//
// Computes, for every (token, slot) pair p routed to expert e,
//   P[p, :] = w[p] * SiLU(Wv[e] x[t])
// as in "MoVA: routing the value vectors, and why the KV cache does not
// notice", section "Where the routing happens" (each selected expert's
// projection passes through SiLU and is weighted by its renormalised score).
//
// At a few tokens per expert the work is a matrix-vector product per active
// expert and HBM-bound: the kernel streams each active expert's n x d weight
// exactly once.  A warp owns a task of two weight rows of one active expert
// and all the tokens routed to it (in chunks of 8): each lane reads 16-byte
// vectors of the rows (no L1 allocation, evict-first in L2, since each row is
// read once) and multiplies them with the matching x vectors (L1/L2 hits).
// Partial sums are reduced by a transposing butterfly, so lane l ends with
// one (row, token) dot product and applies SiLU x weight.  Tasks are spread
// round-robin over all warps of a grid sized to the SM count, so the whole
// GPU streams every active expert in parallel.  Every sum runs in a fixed
// order: results are deterministic.
#include "common.cuh"
#include "internal.h"

namespace mova {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 2;   // weight rows per warp task
constexpr int kTok = 8;    // tokens per chunk

// Transposing butterfly over 16 values per lane: at each step a lane keeps
// one half of its values and trades the other half with its partner, so after
// four steps lane l holds the sum over lanes of value index (l >> 1) & 15 (a
// fifth exchange adds the halves held by lanes l and l ^ 1).
template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V], int lane) {
  static_assert(V == 16, "lane-to-index map assumes 16 values");
  int cnt = V;
  int s = 16;
#pragma unroll
  for (int step = V; step > 1; step >>= 1) {
    const bool upper = (lane & s) != 0;
    const int half = step >> 1;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[i + half];
      const float keep = upper ? v[i + half] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
    s >>= 1;
    cnt = half;
  }
  (void)cnt;
  for (; s >= 1; s >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], s);
  return v[0];
}

template <typename DT>
__global__ void __launch_bounds__(kThreads)
stream_experts_kernel(const DT* __restrict__ x, const DT* __restrict__ Wv,
                      const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                      const int32_t* __restrict__ perm, const float* __restrict__ w32,
                      const int32_t* __restrict__ active, const StatusBlock* __restrict__ sb,
                      int d, int n, int k, float* __restrict__ P) {
  const int nact = sb->num_active;
  const int tasks_per_expert = n / kRows;
  const long long total = static_cast<long long>(nact) * tasks_per_expert;
  const int lane = threadIdx.x & 31;
  const long long gw = (static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * kThreads) >> 5;

  for (long long task = gw; task < total; task += nw) {
    const int a = static_cast<int>(task / tasks_per_expert);
    const int row0 = static_cast<int>(task % tasks_per_expert) * kRows;
    const int e = active[a];
    const int cnt = counts[e];
    const int off = offsets[e];
    const DT* wr0 = Wv + (static_cast<size_t>(e) * n + row0) * d;
    const DT* wr1 = wr0 + d;
    for (int c0 = 0; c0 < cnt; c0 += kTok) {
      const int nt = min(kTok, cnt - c0);
      const DT* xr[kTok];
#pragma unroll
      for (int j = 0; j < kTok; ++j) {
        const int f = perm[off + c0 + min(j, nt - 1)];
        xr[j] = x + static_cast<size_t>(f / k) * d;
      }
      float acc[kRows * kTok];
#pragma unroll
      for (int i = 0; i < kRows * kTok; ++i) acc[i] = 0.f;
#pragma unroll 2
      for (int kk = lane * 8; kk < d; kk += 256) {
        float wa[8], wb[8];
        load8_stream(wr0 + kk, wa);
        load8_stream(wr1 + kk, wb);
#pragma unroll
        for (int j = 0; j < kTok; ++j) {
          if (j < nt) {
            float xv[8];
            load8(xr[j] + kk, xv);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              acc[j] = fmaf(wa[q], xv[q], acc[j]);
              acc[kTok + j] = fmaf(wb[q], xv[q], acc[kTok + j]);
            }
          }
        }
      }
      const float h = transpose_reduce<kRows * kTok>(acc, lane);
      const int vi = (lane >> 1) & 15;
      const int r = vi / kTok;
      const int j = vi % kTok;
      if ((lane & 1) == 0 && j < nt) {
        const int p = off + c0 + j;
        const int f = perm[p];
        P[static_cast<size_t>(p) * n + row0 + r] = w32[f] * siluf_(h);
      }
    }
  }
}

}  // namespace

cudaError_t launch_stream_experts(const void* x, const void* Wv, mova_dtype dt, const int32_t* counts,
                                  const int32_t* offsets, const int32_t* perm, const float* w32,
                                  const int32_t* active, const StatusBlock* sb, int d, int n, int k,
                                  int E, float* P, cudaStream_t stream) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // Upper bound of tasks (all E experts active); the kernel reads the real
  // count of active experts from the status block.
  const long long max_tasks = static_cast<long long>(E) * (n / kRows);
  long long blocks = (max_tasks * 32 + kThreads - 1) / kThreads;
  const long long cap = static_cast<long long>(sms) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (dt == MOVA_BF16) {
    stream_experts_kernel<__nv_bfloat16><<<static_cast<int>(blocks), kThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wv), counts,
        offsets, perm, w32, active, sb, d, n, k, P);
  } else {
    stream_experts_kernel<float><<<static_cast<int>(blocks), kThreads, 0, stream>>>(
        static_cast<const float*>(x), static_cast<const float*>(Wv), counts, offsets, perm, w32,
        active, sb, d, n, k, P);
  }
  return cudaGetLastError();
}

}  // namespace mova
