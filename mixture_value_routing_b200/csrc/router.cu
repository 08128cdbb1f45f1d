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
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "route_select.cuh"
#include "sm100.cuh"

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
  __shared__ float brs[64];

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
  if (tid < 64) brs[tid] = tid < E ? br[tid] : 0.f;

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
  for (int tt = warp; tt < TT; tt += kRouterThreads / 32) {
    const int t = t0 + tt;
    if (t >= T) break;
    int sel_e[8];
    float sel_s[8];
    select_top_k(&part[tt * 64], brs, E, k, lane, sel_e, sel_s);
    const float ssum = sum_k(sel_s, k);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && lane == j) {
        idx_out[(size_t)t * k + j] = sel_e[j];
        w_out[(size_t)t * k + j] = scale * sel_s[j] / ssum;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Decode router (T <= 8), in two parts.
//
// router_logits_kernel: one CTA per (expert, K range), S ranges per expert
// (E * S CTAs, S <= 4).  Each thread takes 8-element chunks of the range:
// the chunk of the expert's router row (requested before
// griddepcontrol.wait: no kernel writes router weights), then the same
// chunk of every token's x, 8 FMAs per token in ascending k.  A transposing
// warp butterfly leaves each token's warp sum in one lane group; the warps'
// sums are added in warp order and stored as part[s][t][e].  Every step has a
// fixed order, so the logits do not depend on timing.  The CTA of (expert 0,
// range 0) also starts the call's status afresh.
//
// The selection and grouping that follow (select_token, group_pairs_warp)
// run either in select_group_kernel (one CTA) or at the start of the
// weight-streaming kernel, which then needs no grouping launch at all.
// ---------------------------------------------------------------------------
constexpr int kDecT = 8;
constexpr int kLogitThreads = kPartThreads;

template <typename XT>
__global__ void __launch_bounds__(kLogitThreads)
router_logits_kernel(const float* __restrict__ Wr, const XT* __restrict__ x, int T, int d, int E,
                     float* __restrict__ part, StatusBlock* __restrict__ sb) {
  __shared__ float red[kLogitThreads / 32][kDecT];
  const int e = blockIdx.x % E;
  const int s = blockIdx.x / E;
  const int S = gridDim.x / E;
  const int chunks = d / 8;
  const int cb = chunks * s / S;
  const int ce = chunks * (s + 1) / S;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const float* wrow = Wr + static_cast<size_t>(e) * d;

  // The first chunk's router weights, in flight during the wait.
  const int c0 = cb + tid;
  float w0[8];
  if (c0 < ce) load8(wrow + 8 * c0, w0);
  pdl_wait();  // x may come from the previous kernel; every output is written after this
  pdl_trigger();
  if (blockIdx.x == 0 && tid == 0 && sb != nullptr) {
    sb->code = 0;
    sb->detail = 0;
    sb->work_next = 0;
  }

  partial_logits_warp(wrow, x, T, d, c0, ce, w0, lane, warp, &red[0][0]);
  __syncthreads();
  if (tid < kDecT) part[(s * kDecT + tid) * 64 + e] = partial_logits_final(&red[0][0], tid);
}

// Selection and grouping of a decode batch by one CTA, from the S partial
// logits: warp t selects token t, warp 0 then groups the pairs.
__global__ void __launch_bounds__(kLogitThreads)
select_group_kernel(const float* __restrict__ part, int S, const float* __restrict__ br, int T, int E,
                    int k, float scale, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                    GroupOut g) {
  __shared__ float lg[kDecT * 64];
  __shared__ float brs[64];
  __shared__ int sel[kDecT * 8];
  __shared__ float wsel[kDecT * 8];
  __shared__ int scratch[128];
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (tid < 64) brs[tid] = tid < E ? br[tid] : 0.f;
  pdl_wait();
  for (int j = tid; j < T * 64; j += kLogitThreads) {
    float v = part[j];
    for (int r = 1; r < S; ++r) v += part[r * kDecT * 64 + j];
    lg[j] = v;
  }
  __syncthreads();
  if (warp < T) select_token(&lg[warp * 64], brs, E, k, scale, warp, lane, sel, wsel, idx_out, w_out);
  if (g.counts == nullptr) return;
  __syncthreads();
  if (warp == 0) {
    const int nact = group_pairs_warp(sel, T * k, E, lane, scratch, g.counts, g.offsets, g.pos, g.perm,
                                      g.active);
    if (lane == 0) g.sb->num_active = nact;
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
  note_launch();
  return cudaLaunchKernelEx(&cfg, router_kernel<XT, TT>, static_cast<const XT*>(x), Wr, br, T, d,
                            E, k, scale, idx, w);
}

template <typename XT>
cudaError_t launch_logits_t(const void* x, const float* Wr, int T, int d, int E, int S, float* part,
                            StatusBlock* sb, cudaStream_t stream) {
  return launch_pdl(router_logits_kernel<XT>, dim3(static_cast<unsigned>(E * S)), dim3(kLogitThreads), 0,
                    stream, Wr, static_cast<const XT*>(x), T, d, E, part, sb);
}

}  // namespace

cudaError_t launch_router(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                          int d, int E, int k, float scale, int32_t* idx, float* w,
                          const GroupOut* g, bool* grouped, int partitions, cudaStream_t stream) {
  if (grouped) *grouped = false;
  if (T <= 0) return cudaSuccess;
  if (T <= kFusedRouterMaxT && g != nullptr && g->logits != nullptr) {
    int S = 0;
    cudaError_t err = launch_router_logits(x, x_dt, Wr, T, d, E, partitions, g->logits, &S, g->sb, stream);
    if (err != cudaSuccess) return err;
    if (grouped) *grouped = true;
    return launch_select_group(g->logits, S, br, T, E, k, scale, idx, w, g, stream);
  }
  const bool small = T <= 64;
  const int TT = small ? 8 : 32;
  const int ntiles = (T + TT - 1) / TT;
  // Enough CTAs to cover the SMs twice; at most 8 (portable cluster size).
  int ks = (2 * sm_count() + ntiles - 1) / ntiles;
  if (ks > 8) ks = 8;
  if (ks < 1) ks = 1;
  if (ks > d / kRouterKC) ks = d / kRouterKC;
  // Two router partitions: exactly two ranks, rank 0 summing j < d/2 and
  // rank 1 the rest; rank 0 adds rank 1's fp32 partial to its own.
  if (partitions == 2) ks = 2;
  if (x_dt == MOVA_BF16) {
    return small ? launch_router_t<__nv_bfloat16, 8>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream)
                 : launch_router_t<__nv_bfloat16, 32>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream);
  }
  return small ? launch_router_t<float, 8>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream)
               : launch_router_t<float, 32>(x, Wr, br, T, d, E, k, scale, idx, w, ks, stream);
}

int logit_splits(int d, int E) {
  int S = 1;
  while (S < kMaxLogitSplits && E * S * 2 <= sm_count() && d / 8 >= 2 * S * kLogitThreads / 4) S *= 2;
  return S;
}

// Two router partitions: exactly two K ranges, the halves of d; the
// selection adds their fp32 partial logits in range order.
int decode_logit_splits(int d, int E, int partitions) { return partitions == 2 ? 2 : logit_splits(d, E); }

cudaError_t launch_router_logits(const void* x, mova_dtype x_dt, const float* Wr, int T, int d, int E,
                                 int partitions, float* part, int* S_out, StatusBlock* sb,
                                 cudaStream_t stream) {
  if (T <= 0 || T > kDecT) return cudaErrorInvalidValue;
  const int S = decode_logit_splits(d, E, partitions);
  *S_out = S;
  return x_dt == MOVA_BF16 ? launch_logits_t<__nv_bfloat16>(x, Wr, T, d, E, S, part, sb, stream)
                           : launch_logits_t<float>(x, Wr, T, d, E, S, part, sb, stream);
}

cudaError_t launch_select_group(const float* part, int S, const float* br, int T, int E, int k, float scale,
                                int32_t* idx, float* w, const GroupOut* g, cudaStream_t stream) {
  GroupOut go{};
  if (g != nullptr) go = *g;
  return launch_pdl(select_group_kernel, dim3(1), dim3(kLogitThreads), 0, stream, part, S, br, T, E, k, scale,
                    idx, w, go);
}

}  // namespace mova
