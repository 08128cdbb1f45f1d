// Value router: fp32 logits, sigmoid gate, bias-assisted top-k, renormalise,
// scale.  Follows "MoVA: routing the value vectors, and why the KV cache does
// not notice", section "Where the routing happens": the router's linear map
// runs without its bias; the bias is handed to the gate and only steers the
// selection; the k sigmoid scores of the selected experts are renormalised
// and multiplied by the scaling factor (2.5 in the released model).
//
// Design (B200): a CTA owns a tile of TT tokens and all E <= 64 experts.  A
// thread-block cluster of KS CTAs splits the d-long dot products into KS
// ranges of K (so a decode batch of 8 tokens spreads its 655 KB weight read
// over KS SMs); partial logits meet in CTA rank 0 through distributed shared
// memory and are summed in rank order, so results are deterministic.  Then
// one warp per token holds two experts per lane, forms the biased scores in
// registers and runs k rounds of a warp arg-max (ties -> lower index).
#include <cooperative_groups.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace mova {

namespace {

__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  uint2 u = *reinterpret_cast<const uint2*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
  float2 a = __bfloat1622float2(h[0]);
  float2 b = __bfloat1622float2(h[1]);
  return make_float4(a.x, a.y, b.x, b.y);
}

constexpr int kRouterThreads = 128;
constexpr int kRouterKC = 32;  // K elements per shared-memory chunk

template <typename XT, int TT>
__global__ void __launch_bounds__(kRouterThreads)
router_kernel(const XT* __restrict__ x, const float* __restrict__ Wr, const float* __restrict__ br,
              int T, int d, int E, int k, float scale, int32_t* __restrict__ idx_out,
              float* __restrict__ w_out) {
  constexpr int KC = kRouterKC;
  constexpr int TPT = TT / 8;  // tokens per thread (8 token groups x 16 expert groups)
  __shared__ __align__(16) float xs[TT][KC + 4];
  __shared__ __align__(16) float wsm[64][KC + 4];
  __shared__ __align__(16) float part[TT * 64];

  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int ks = gridDim.x;  // the cluster spans blockIdx.x
  const int rank = blockIdx.x;
  const int t0 = blockIdx.y * TT;
  const int nchunks = d / KC;
  const int c_begin = rank * nchunks / ks;
  const int c_end = (rank + 1) * nchunks / ks;
  const int tg = tid >> 4;
  const int eg = tid & 15;

  float acc[TPT][4];
#pragma unroll
  for (int i = 0; i < TPT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;

  for (int c = c_begin; c < c_end; ++c) {
    const int k0 = c * KC;
    for (int i = tid; i < TT * (KC / 4); i += kRouterThreads) {
      const int r = i / (KC / 4);
      const int cc = (i % (KC / 4)) * 4;
      const int t = t0 + r;
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (t < T) val = load4(x + (size_t)t * d + k0 + cc);
      *reinterpret_cast<float4*>(&xs[r][cc]) = val;
    }
    for (int i = tid; i < 64 * (KC / 4); i += kRouterThreads) {
      const int r = i / (KC / 4);
      const int cc = (i % (KC / 4)) * 4;
      float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < E) val = *reinterpret_cast<const float4*>(Wr + (size_t)r * d + k0 + cc);
      *reinterpret_cast<float4*>(&wsm[r][cc]) = val;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < KC; kk += 4) {
      float4 wv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[j] = *reinterpret_cast<const float4*>(&wsm[eg + 16 * j][kk]);
#pragma unroll
      for (int i = 0; i < TPT; ++i) {
        const float4 xv = *reinterpret_cast<const float4*>(&xs[tg * TPT + i][kk]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(xv.x, wv[j].x, acc[i][j]);
          acc[i][j] = fmaf(xv.y, wv[j].y, acc[i][j]);
          acc[i][j] = fmaf(xv.z, wv[j].z, acc[i][j]);
          acc[i][j] = fmaf(xv.w, wv[j].w, acc[i][j]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < TPT; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) part[(tg * TPT + i) * 64 + eg + 16 * j] = acc[i][j];

  cluster.sync();
  if (ks > 1 && rank == 0) {
    // Sum the partial logits of the cluster's CTAs in rank order.
    for (int i = tid; i < TT * 64; i += kRouterThreads) {
      float s = part[i];
      for (int r = 1; r < ks; ++r) s += cluster.map_shared_rank(part, r)[i];
      part[i] = s;
    }
  }
  cluster.sync();  // the other CTAs' shared memory stays alive until here
  if (rank != 0) return;

  const int warp = tid >> 5;
  const int lane = tid & 31;
  const float NEG = -INFINITY;
  for (int tt = warp; tt < TT; tt += kRouterThreads / 32) {
    const int t = t0 + tt;
    if (t >= T) break;
    // Two experts per lane.  A candidate is (biased score, key); the key is
    // the expert index, plus 64 once the expert is taken or does not exist,
    // so such candidates lose every tie against a live expert (NaN scores are
    // mapped to -inf and can never displace a finite one).
    const int e0 = lane, e1 = lane + 32;
    float s0 = 0.f, s1 = 0.f, b0 = NEG, b1 = NEG;
    int key0 = e0 + 64, key1 = e1 + 64;
    if (e0 < E) {
      s0 = sigmoidf_(part[tt * 64 + e0]);
      b0 = s0 + br[e0];
      if (!(b0 == b0)) b0 = NEG;
      key0 = e0;
    }
    if (e1 < E) {
      s1 = sigmoidf_(part[tt * 64 + e1]);
      b1 = s1 + br[e1];
      if (!(b1 == b1)) b1 = NEG;
      key1 = e1;
    }
    int sel_e[8];
    float sel_s[8];
    float ssum = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        // Lane-local best, then a warp arg-max under the total order
        // (score descending, key ascending): ties go to the lower index.
        float bb = b0, bs = s0;
        int be = key0;
        if (b1 > b0 || (b1 == b0 && key1 < key0)) { bb = b1; bs = s1; be = key1; }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const float ob = __shfl_xor_sync(0xffffffffu, bb, off);
          const float os = __shfl_xor_sync(0xffffffffu, bs, off);
          const int oe = __shfl_xor_sync(0xffffffffu, be, off);
          if (ob > bb || (ob == bb && oe < be)) { bb = ob; bs = os; be = oe; }
        }
        be &= 63;  // always a live expert: k <= E
        sel_e[j] = be;
        sel_s[j] = bs;
        ssum += bs;
        if (be == e0) { b0 = NEG; key0 = e0 + 64; }
        if (be == e1) { b1 = NEG; key1 = e1 + 64; }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && lane == j) {
        idx_out[(size_t)t * k + j] = sel_e[j];
        w_out[(size_t)t * k + j] = scale * sel_s[j] / ssum;
      }
    }
  }
}

template <typename XT, int TT>
cudaError_t launch_router_t(const void* x, const float* Wr, const float* br, int T, int d, int E,
                            int k, float scale, int32_t* idx, float* w, int ks,
                            cudaStream_t stream) {
  const int ntiles = (T + TT - 1) / TT;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ks, ntiles, 1);
  cfg.blockDim = dim3(kRouterThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = ks;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_kernel<XT, TT>, static_cast<const XT*>(x), Wr, br, T, d,
                            E, k, scale, idx, w);
}

}  // namespace

cudaError_t launch_router(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                          int d, int E, int k, float scale, int32_t* idx, float* w,
                          cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const bool small = T <= 64;
  const int TT = small ? 8 : 32;
  const int ntiles = (T + TT - 1) / TT;
  // Enough CTAs to cover the SMs twice; at most 8 (portable cluster size).
  int ks = (2 * 148 + ntiles - 1) / ntiles;
  if (ks > 8) ks = 8;
  if (ks < 1) ks = 1;
  if (ks > d / kRouterKC) ks = d / kRouterKC;
  if (x_dt == MOVA_BF16) {
    return small ? launch_router_t<__nv_bfloat16, 8>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream)
                 : launch_router_t<__nv_bfloat16, 32>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream);
  }
  return small ? launch_router_t<float, 8>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream)
               : launch_router_t<float, 32>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream);
}

}  // namespace mova
