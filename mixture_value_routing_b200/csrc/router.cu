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

// Gate and selection of one token by one warp.  lg: the token's E logits (in
// shared memory).  Lane l holds experts l and l + 32.  A candidate is (biased
// score, key); the key is the expert index, plus 64 once the expert is taken
// or does not exist, so such candidates lose every tie against a live expert
// (NaN scores are mapped to -inf and can never displace a finite one).  k
// rounds of a warp arg-max under the total order (score descending, key
// ascending) pick the experts: ties go to the lower index.  On return every
// lane holds the same sel_e / sel_s (unbiased sigmoid scores) for j < k.
__device__ __forceinline__ void select_top_k(const float* lg, const float* __restrict__ br, int E,
                                             int k, int lane, int (&sel_e)[8], float (&sel_s)[8]) {
  const float NEG = -INFINITY;
  const int e0 = lane, e1 = lane + 32;
  float s0 = 0.f, s1 = 0.f, b0 = NEG, b1 = NEG;
  int key0 = e0 + 64, key1 = e1 + 64;
  if (e0 < E) {
    s0 = sigmoidf_(lg[e0]);
    b0 = s0 + br[e0];
    if (!(b0 == b0)) b0 = NEG;
    key0 = e0;
  }
  if (e1 < E) {
    s1 = sigmoidf_(lg[e1]);
    b1 = s1 + br[e1];
    if (!(b1 == b1)) b1 = NEG;
    key1 = e1;
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
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
      if (be == e0) { b0 = NEG; key0 = e0 + 64; }
      if (be == e1) { b1 = NEG; key1 = e1 + 64; }
    }
  }
}

// Sum of the k selected scores in slot order.
__device__ __forceinline__ float sum_k(const float (&s)[8], int k) {
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) acc += s[j];
  return acc;
}

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
  for (int tt = warp; tt < TT; tt += kRouterThreads / 32) {
    const int t = t0 + tt;
    if (t >= T) break;
    int sel_e[8];
    float sel_s[8];
    select_top_k(&part[tt * 64], br, E, k, lane, sel_e, sel_s);
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
// Decode router (T <= 8): one cluster of 8 CTAs x 8 warps, one warp per
// expert.  Each warp issues its whole router row (d fp32) as 16-byte loads at
// once and dots it with every token's x (L1/L2 hits), so the 655 KB router
// read is spread over 64 warps with all loads in flight.  Partial sums are
// reduced across lanes in a fixed butterfly order; each warp writes its
// expert's T logits into CTA rank 0's shared memory (distributed shared
// memory).  Rank 0 then selects per token (warp per token) and, as T*k <= 64
// pairs, also groups the pairs by expert in the same kernel (stable counting
// sort by one warp), so a decode step needs no separate grouping launch.
// ---------------------------------------------------------------------------
constexpr int kSmallT = 8;
constexpr int kSmallWarps = 8;
constexpr size_t kSmallRouterSmem = 160 * 1024;  // largest staged x tile

constexpr int kSmallQ = 4;                        // warps per expert (K quarters)
constexpr int kSmallThreads = kSmallWarps * kSmallQ * 32;
constexpr int kSmallCH = 5;                       // float4 loads in flight per lane and pass

template <typename XT>
__global__ void __launch_bounds__(kSmallThreads)
router_small_kernel(const XT* __restrict__ x, const float* __restrict__ Wr,
                    const float* __restrict__ br, int T, int d, int E, int k, float scale,
                    int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                    GroupOut g) {
  extern __shared__ __align__(16) uint8_t xsm[];  // the T x d tokens, as stored
  __shared__ float logits[kSmallT][64];
  __shared__ float part[kSmallQ][kSmallWarps][kSmallT];
  __shared__ int sel[kSmallT * 8];
  cg::cluster_group cluster = cg::this_cluster();
  const XT* xs = reinterpret_cast<const XT*>(xsm);
  const int rank = blockIdx.x;  // 8 CTAs per cluster, 8 experts per CTA
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int el = warp >> 2;     // expert within the CTA
  const int q = warp & 3;       // K quarter
  const int e = rank * kSmallWarps + el;
  float* rlog = cluster.map_shared_rank(&logits[0][0], 0);
  // Every CTA of the cluster must have started before shared memory of
  // another CTA is written: arrive now, wait just before the remote stores.
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");

  // K is cut into chunks of 128 (32 lanes x float4); quarter q owns a
  // contiguous run of chunks.
  const int nchunk = (d + 127) / 128;
  const int cb = nchunk * q / kSmallQ;
  const int ce = nchunk * (q + 1) / kSmallQ;
  const float* wrow = Wr + static_cast<size_t>(min(e, E - 1)) * d;
  float4 wv[kSmallCH];
#pragma unroll
  for (int i = 0; i < kSmallCH; ++i) {
    const int kk = (cb + i) * 128 + lane * 4;
    wv[i] = (cb + i < ce && kk < d) ? __ldg(reinterpret_cast<const float4*>(wrow + kk))
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  {
    const int nvec = static_cast<int>(static_cast<size_t>(T) * d * sizeof(XT) / 16);
    const uint4* src = reinterpret_cast<const uint4*>(x);
    uint4* dst = reinterpret_cast<uint4*>(xsm);
    for (int i = threadIdx.x; i < nvec; i += kSmallThreads) dst[i] = src[i];
  }
  __syncthreads();

  float acc[kSmallT];
#pragma unroll
  for (int t = 0; t < kSmallT; ++t) acc[t] = 0.f;
  for (int c0 = cb; c0 < ce; c0 += kSmallCH) {
    if (c0 > cb) {
#pragma unroll
      for (int i = 0; i < kSmallCH; ++i) {
        const int kk = (c0 + i) * 128 + lane * 4;
        wv[i] = (c0 + i < ce && kk < d) ? __ldg(reinterpret_cast<const float4*>(wrow + kk))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int t = 0; t < kSmallT; ++t) {
      if (t < T) {
#pragma unroll
        for (int i = 0; i < kSmallCH; ++i) {
          const int kk = (c0 + i) * 128 + lane * 4;
          if (c0 + i < ce && kk < d) {
            const float4 xv = load4(xs + static_cast<size_t>(t) * d + kk);
            acc[t] = fmaf(xv.x, wv[i].x, acc[t]);
            acc[t] = fmaf(xv.y, wv[i].y, acc[t]);
            acc[t] = fmaf(xv.z, wv[i].z, acc[t]);
            acc[t] = fmaf(xv.w, wv[i].w, acc[t]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < kSmallT; ++t) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < kSmallT; ++t) part[q][el][t] = acc[t];
  }
  __syncthreads();
  asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
  // The four K quarters of each expert, summed in order, go to rank 0.
  if (threadIdx.x < kSmallWarps * kSmallT) {
    const int ee = threadIdx.x / kSmallT;
    const int t = threadIdx.x % kSmallT;
    const int eg = rank * kSmallWarps + ee;
    if (eg < E) {
      float v = part[0][ee][t];
#pragma unroll
      for (int qq = 1; qq < kSmallQ; ++qq) v += part[qq][ee][t];
      rlog[t * 64 + eg] = v;
    }
  }
  cluster.sync();
  if (rank != 0) return;

  // Selection: warp t handles token t.
  if (warp < T) {
    const int t = warp;
    float ws_[8];
    int es_[8];
    select_top_k(&logits[t][0], br, E, k, lane, es_, ws_);
    const float ssum = sum_k(ws_, k);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k && lane == j) {
        idx_out[t * k + j] = es_[j];
        w_out[t * k + j] = scale * ws_[j] / ssum;
        sel[t * k + j] = es_[j];
      }
    }
  }
  if (g.counts == nullptr) return;
  __syncthreads();
  if (warp != 0) return;
  // Grouping of the N = T*k <= 64 pairs by one warp (stable counting sort).
  const int N = T * k;
  const int f0 = lane, f1 = lane + 32;
  const int ef0 = (f0 < N) ? sel[f0] : -1;
  const int ef1 = (f1 < N) ? sel[f1] : -1;
  int rank0 = 0, rank1 = 0, cnt0 = 0, cnt1 = 0;
  for (int f = 0; f < N; ++f) {
    const int ef = sel[f];
    rank0 += (f < f0 && ef == ef0);
    rank1 += (f < f1 && ef == ef1);
    cnt0 += (ef == lane);
    cnt1 += (ef == lane + 32);
  }
  // Exclusive scan of the counts over experts lane, lane+32.
  int inc0 = cnt0;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc0, off);
    if (lane >= off) inc0 += y;
  }
  const int tot0 = __shfl_sync(0xffffffffu, inc0, 31);
  int inc1 = cnt1;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc1, off);
    if (lane >= off) inc1 += y;
  }
  const int ex0 = inc0 - cnt0;
  const int ex1 = tot0 + inc1 - cnt1;
  if (lane < E) { g.counts[lane] = cnt0; g.offsets[lane] = ex0; }
  if (lane + 32 < E) { g.counts[lane + 32] = cnt1; g.offsets[lane + 32] = ex1; }
  if (lane == 0) g.offsets[E] = N;
  __shared__ int offs[64];
  offs[lane] = ex0;
  offs[lane + 32] = ex1;
  __syncwarp();
  if (f0 < N) { const int p = offs[ef0] + rank0; g.pos[f0] = p; g.perm[p] = f0; }
  if (f1 < N) { const int p = offs[ef1] + rank1; g.pos[f1] = p; g.perm[p] = f1; }
  const bool a0 = lane < E && cnt0 > 0;
  const bool a1 = lane + 32 < E && cnt1 > 0;
  const unsigned m0 = __ballot_sync(0xffffffffu, a0);
  const unsigned m1 = __ballot_sync(0xffffffffu, a1);
  const unsigned lt = (1u << lane) - 1u;
  if (a0) g.active[__popc(m0 & lt)] = lane;
  if (a1) g.active[__popc(m0) + __popc(m1 & lt)] = lane + 32;
  if (lane == 0) {
    g.sb->code = 0;
    g.sb->detail = 0;
    g.sb->num_active = __popc(m0) + __popc(m1);
    g.sb->work_next = 0;
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

template <typename XT>
cudaError_t launch_router_small(const void* x, const float* Wr, const float* br, int T, int d,
                                int E, int k, float scale, int32_t* idx, float* w, GroupOut g,
                                cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(T) * d * sizeof(XT);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(router_small_kernel<XT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kSmallRouterSmem));
    if (err != cudaSuccess) return err;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(8, 1, 1);
  cfg.blockDim = dim3(kSmallThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 8;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, router_small_kernel<XT>, static_cast<const XT*>(x), Wr, br, T,
                            d, E, k, scale, idx, w, g);
}

}  // namespace

cudaError_t launch_router(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                          int d, int E, int k, float scale, int32_t* idx, float* w,
                          const GroupOut* g, bool* grouped, cudaStream_t stream) {
  if (grouped) *grouped = false;
  if (T <= 0) return cudaSuccess;
  const size_t xbytes = static_cast<size_t>(T) * d * (x_dt == MOVA_BF16 ? 2 : 4);
  if (T <= kFusedRouterMaxT && xbytes <= kSmallRouterSmem) {
    GroupOut go{};
    if (g != nullptr) go = *g;
    if (grouped) *grouped = (g != nullptr);
    return x_dt == MOVA_BF16
               ? launch_router_small<__nv_bfloat16>(x, Wr, br, T, d, E, k, scale, idx, w, go, stream)
               : launch_router_small<float>(x, Wr, br, T, d, E, k, scale, idx, w, go, stream);
  }
  const bool small = T <= 64;
  const int TT = small ? 8 : 32;
  const int ntiles = (T + TT - 1) / TT;
  // Enough CTAs to cover the SMs twice; at most 8 (portable cluster size).
  int ks = (2 * sm_count() + ntiles - 1) / ntiles;
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
