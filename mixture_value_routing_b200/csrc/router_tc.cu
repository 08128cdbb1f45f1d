// Tensor-core router for large bf16 batches.
//
// "MoVA: routing the value vectors, and why the KV cache does not notice",
// section "Where the routing happens": logits = x Wr^T (no bias), sigmoid
// gate, the bias steers a top-k selection, the k scores are renormalised and
// scaled.  At prefill sizes the logits are a dense T x 2560 x 64 contraction,
// so they run on tcgen05 tensor cores with fp32 accumulation:
//
//   * x is bf16, so every product x_j * Wr[e, j] is formed exactly if Wr is
//     bf16 too.  The fp32 router weight is therefore split exactly into three
//     bf16 planes, Wr = hi + mid + lo (8 + 8 + 8 significand bits cover fp32's
//     24; each plane is the round-to-nearest bf16 of what the previous ones
//     left), and the router runs as one GEMM against the 3E = 192 plane rows.
//     logits[e] = (acc_hi[e] + acc_mid[e]) + acc_lo[e]: the same products as
//     an fp32 dot product, accumulated in fp32 in another order.
//   * One SM pair (a two-CTA cluster) per 256 tokens: each CTA's TMA warp
//     streams its 128 x 64 token tile and its half (96 rows) of the 192 x 64
//     plane tile (128-byte swizzle) through 7 stages of 28 KB, so a CTA
//     streams 30% fewer bytes than with all plane rows in every CTA; the even
//     CTA issues tcgen05.mma.cta_group::2 (M = 256 tokens, N = 192, K = 16),
//     which accumulates each CTA's 128 tokens in its own tensor memory.
//     Sixteen epilogue warps per CTA, four per 32-token lane quarter, each
//     over 16 experts: a thread forms its token's 16 logits, sigmoid scores
//     and the top k of those 16 in registers; one thread per token then
//     merges the four lists and writes idx / w, plus the 128-token tile's
//     expert histogram for the grouping.  (With one thread per token over
//     all 64 experts, the epilogue took twice as long as the main loop.)
// Every wait is bounded (MOVA_ERR_TIMEOUT, then drain and free).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mova {

namespace {

constexpr int RM = 128;  // tokens per CTA (256 per SM pair)
constexpr int RN = 192;  // 3 planes x 64 experts (96 plane rows in each CTA of the pair)
constexpr int RK = 64;
constexpr int kRStages = 7;
constexpr int kRABytes = RM * RK * 2;
constexpr int kRBBytes = (RN / 2) * RK * 2;
constexpr int kRStageBytes = kRABytes + kRBBytes;
constexpr int kRThreads = 18 * 32;  // warp 0 TMA, warp 1 MMA, warps 2-17 epilogue
constexpr uint32_t kRTmemCols = 256;

struct __align__(1024) RSmem {
  uint8_t stage[kRStages][kRStageBytes];
  uint64_t full[kRStages];
  uint64_t empty[kRStages];
  uint64_t tmem_full;
  uint32_t tmem_base;
  int abort;
  int hist[64];
  float br[64];
};

// Exact split of an fp32 value into three bf16 values summing to it.
// Each thread handles up to kSplitPer elements of Wr (8 consecutive floats
// per step).  The router weights are read and split while the previous
// kernel on the stream may still run (launched with programmatic dependent
// launch; no kernel writes router weights), but the planes are stored only
// after griddepcontrol.wait: they live in the caller's workspace, where the
// previous call's kernels may still be reading other data at the same
// offsets (the workspace layout depends on the call's sizes).
constexpr int kSplitPer = 2;  // 8-element groups per thread
__global__ void __launch_bounds__(256)
split_router_kernel(const float* __restrict__ Wr, int E, int d, __nv_bfloat16* __restrict__ W3) {
  const int groups = 64 * d / 8;
  uint4 hi[kSplitPer], mid[kSplitPer], lo[kSplitPer];
  int gi[kSplitPer];
#pragma unroll
  for (int q = 0; q < kSplitPer; ++q) {
    const int g = (blockIdx.x * kSplitPer + q) * 256 + threadIdx.x;
    gi[q] = g;
    if (g >= groups) continue;
    const int e = g * 8 / d;
    float v[8];
    if (e < E) {
      load8(Wr + static_cast<size_t>(g) * 8, v);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = 0.f;
    }
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi[q]);
    __nv_bfloat162* m = reinterpret_cast<__nv_bfloat162*>(&mid[q]);
    __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo[q]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float a = v[2 * i], b = v[2 * i + 1];
      const __nv_bfloat162 ha = __floats2bfloat162_rn(a, b);
      a -= __low2float(ha);
      b -= __high2float(ha);
      const __nv_bfloat162 ma = __floats2bfloat162_rn(a, b);
      a -= __low2float(ma);
      b -= __high2float(ma);
      h[i] = ha;
      m[i] = ma;
      l[i] = __floats2bfloat162_rn(a, b);
    }
  }
  pdl_wait();  // every kernel before this one on the stream has completed
  const size_t plane = static_cast<size_t>(64) * d / 8;  // uint4 per plane
  uint4* W = reinterpret_cast<uint4*>(W3);
#pragma unroll
  for (int q = 0; q < kSplitPer; ++q) {
    if (gi[q] >= groups) continue;
    W[gi[q]] = hi[q];
    W[plane + gi[q]] = mid[q];
    W[2 * plane + gi[q]] = lo[q];
  }
}

// 18 warps: sub-partitions 0 and 1 hold five warps each, so at most
// 16384 / (5 * 32) -> 96 registers per thread.
__global__ void __maxnreg__(96)
router_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                 const float* __restrict__ br, int T, int d, int E, int k, float scale,
                 int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                 int32_t* __restrict__ tile_counts, StatusBlock* __restrict__ sb, int parts) {
  extern __shared__ uint8_t smem_raw[];
  RSmem& S = *reinterpret_cast<RSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int nk = d / RK;
  const int t0 = blockIdx.x * RM;  // this CTA's 128 tokens (the pair's M = 256)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    mbar_init(&S.tmem_full, 1);
    S.abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 64) {
    S.hist[threadIdx.x] = 0;
    S.br[threadIdx.x] = (threadIdx.x < E) ? br[threadIdx.x] : 0.f;
  }
  // Two router partitions keep a second accumulator (columns 256..447) for
  // the second half of d.
  const uint32_t tmem_cols = parts == 2 ? 2 * kRTmemCols : kRTmemCols;
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, tmem_cols);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the plane split of this call is complete
  tc_fence_before();
  cluster_sync_all();  // barriers and tensor memory of both CTAs are ready
  tc_fence_after();

  if (warp == 0) {
    // The whole warp runs the loop; one elected lane issues the copies: this
    // CTA's 128 token rows and its half of the 192 plane rows, completing on
    // the even CTA's stage barrier (which declares both CTAs' bytes).
    const uint32_t full0_cl = mapa_shared(smem_u32(&S.full[0]), 0);
    int s = 0;
    uint32_t phase = 0;
    for (int kb = 0; kb < nk; ++kb) {
      if (kb >= kRStages && !__all_sync(0xffffffffu, mbar_wait(&S.empty[s], phase ^ 1))) {
        if (lane == 0) {
          raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
          S.abort = 1;
        }
        break;
      }
      if (elect_one()) {
        const uint32_t full_cl = full0_cl + static_cast<uint32_t>(s) * 8u;
        if (rank == 0) mbar_arrive_expect_tx(&S.full[s], 2 * kRStageBytes);
        tma_load_2d_pair(S.stage[s], &tmap_x, kb * RK, t0, full_cl);
        tma_load_2d_pair(S.stage[s] + kRABytes, &tmap_w, kb * RK, static_cast<int>(rank) * (RN / 2), full_cl);
      }
      __syncwarp();
      if (++s == kRStages) {
        s = 0;
        phase ^= 1;
      }
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // The whole warp runs the loop; one elected lane issues the pair's
      // MMAs (M = 256 tokens, N = 192 plane rows: 96 from each CTA) and
      // commits to both CTAs' barriers.
      const uint32_t idesc = idesc_bf16_f32(2 * RM, RN);
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(S.stage[0]));
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(S.stage[0]) + kRABytes);
      constexpr uint32_t kStageDesc = kRStageBytes >> 4;
      bool ok = true;
      int s = 0;
      uint32_t phase = 0;
      const int khalf = parts == 2 ? nk / 2 : nk;
      for (int kb = 0; kb < nk; ++kb) {
        if (!__all_sync(0xffffffffu, mbar_wait(&S.full[s], phase))) {
          if (lane == 0) {
            raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
            S.abort = 1;
          }
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t da = adesc0 + static_cast<uint64_t>(s) * kStageDesc;
        const uint64_t db = bdesc0 + static_cast<uint64_t>(s) * kStageDesc;
        const bool second = kb >= khalf;
        const uint32_t d_tmem = S.tmem_base + (second ? kRTmemCols : 0u);
        const int kl = second ? kb - khalf : kb;  // k-step within its partition
        if (elect_one()) {
#pragma unroll
          for (int k16 = 0; k16 < RK / 16; ++k16)
            tc_mma_bf16_pair(d_tmem, da + 2 * k16, db + 2 * k16, idesc, (kl | k16) != 0);
          tc_commit_pair_both(&S.empty[s]);
        }
        __syncwarp();
        if (++s == kRStages) {
          s = 0;
          phase ^= 1;
        }
      }
      if (ok && elect_one()) tc_commit_pair_both(&S.tmem_full);
      __syncwarp();
    }
  } else {
    // Epilogue: warp w reads TMEM lanes 32 * (w % 4) .. +31 (tokens) and the
    // hi / mid / lo columns of experts 16 g .. 16 g + 15, g = (w - 2) / 4:
    // the warps of one lane quarter split the 64 experts four ways.  Each
    // thread forms its 16 logits and scores and the top k of its 16 experts
    // in the selection order (highest biased score first, ties to the lower
    // index); then one thread per token merges the four lists.
    const int q = warp & 3;
    const int g = (warp - 2) >> 2;
    const int tl = q * 32 + lane;  // token within the CTA
    // Candidate lists in the (drained) stage ring: [group][rank][token].
    float* cb = reinterpret_cast<float*>(S.stage[0]);
    float* cs = cb + 4 * 8 * RM;
    int* ce = reinterpret_cast<int*>(cs + 4 * 8 * RM);
    if (mbar_wait(&S.tmem_full, 0)) {
      tc_fence_after();
      const uint32_t tb = S.tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(g * 16);
      float sc[16];
      {
        uint32_t hi[16], mid[16], lo[16];
        tmem_ld_16(tb, hi);
        tmem_ld_16(tb + 64, mid);
        tmem_ld_16(tb + 128, lo);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          sc[j] = (__uint_as_float(hi[j]) + __uint_as_float(mid[j])) + __uint_as_float(lo[j]);
        if (parts == 2) {
          // Second partition: its own fp32 partial, added after the first.
          tmem_ld_16(tb + kRTmemCols, hi);
          tmem_ld_16(tb + kRTmemCols + 64, mid);
          tmem_ld_16(tb + kRTmemCols + 128, lo);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            sc[j] += (__uint_as_float(hi[j]) + __uint_as_float(mid[j])) + __uint_as_float(lo[j]);
        }
      }
      tc_fence_before();
      // Sigmoid scores (in place); the biased score s + br steers the
      // selection only, NaN never wins.
      float bs[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        sc[j] = sigmoidf_(sc[j]);
        const float b = sc[j] + S.br[g * 16 + j];
        bs[j] = b == b ? b : -INFINITY;
      }
      const int live = min(max(E - g * 16, 0), 16);  // this group's experts below E
      uint32_t taken = 0;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r < k && r < live) {
          int be = -1;
          float bb = 0.f, bsv = 0.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (j < live && !((taken >> j) & 1u) && (be < 0 || bs[j] > bb)) {
              be = j;
              bb = bs[j];
              bsv = sc[j];
            }
          }
          taken |= 1u << be;
          const int o = (g * 8 + r) * RM + tl;
          cb[o] = bb;
          cs[o] = bsv;
          ce[o] = g * 16 + be;
        }
      }
    } else {
      raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
      S.abort = 1;
    }
    asm volatile("bar.sync 1, 512;" ::: "memory");  // the 16 epilogue warps: every list is written
    const int t = t0 + tl;
    if (g == 0 && t < T && !*reinterpret_cast<volatile int*>(&S.abort)) {
      // Merge: repeatedly take the best head of the four lists (strictly
      // greater biased score; equal scores keep the lower group, i.e. the
      // lower expert index, as the lists are in ascending expert ranges).
      int nlen[4], head[4];
#pragma unroll
      for (int gg = 0; gg < 4; ++gg) {
        nlen[gg] = min(k, min(max(E - gg * 16, 0), 16));
        head[gg] = 0;
      }
      int sel[8];
      float ssel[8];
      float ssum = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k) {
          int bg = -1;
          float bb = 0.f;
#pragma unroll
          for (int gg = 0; gg < 4; ++gg) {
            if (head[gg] < nlen[gg]) {
              const float b = cb[(gg * 8 + head[gg]) * RM + tl];
              if (bg < 0 || b > bb) {
                bg = gg;
                bb = b;
              }
            }
          }
          int o = 0;
#pragma unroll
          for (int gg = 0; gg < 4; ++gg)
            if (gg == bg) {
              o = (gg * 8 + head[gg]) * RM + tl;
              ++head[gg];
            }
          sel[j] = ce[o];
          ssel[j] = cs[o];
          ssum += ssel[j];
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < k) {
          idx_out[static_cast<size_t>(t) * k + j] = sel[j];
          w_out[static_cast<size_t>(t) * k + j] = scale * ssel[j] / ssum;
          atomicAdd(&S.hist[sel[j]], 1);
        }
      }
    }
  }
  __syncthreads();
  if (tile_counts != nullptr && threadIdx.x < 64 && t0 < T)
    tile_counts[blockIdx.x * 64 + threadIdx.x] = S.hist[threadIdx.x];
  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while the pair may still touch its memory
  if (S.abort && threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) mbar_wait(&S.empty[s], 0);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(S.tmem_base, tmem_cols);
  }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

size_t router_planes_bytes(int d) { return static_cast<size_t>(RN) * d * 2; }

cudaError_t launch_split_router(const float* Wr, int E, int d, __nv_bfloat16* planes, cudaStream_t stream) {
  const int split_blocks = (64 * d / 8 + 256 * kSplitPer - 1) / (256 * kSplitPer);
  return launch_pdl(split_router_kernel, dim3(split_blocks), dim3(256), 0, stream, Wr, E, d, planes);
}

cudaError_t launch_router_tc(const void* x, const float* Wr, const float* br, int T, int d, int E,
                             int k, float scale, int partitions, int32_t* idx, float* w,
                             int32_t* tile_counts, __nv_bfloat16* planes, const __nv_bfloat16* prepared,
                             StatusBlock* sb, cudaStream_t stream) {
  void* fp = encode_tiled_fn();
  if (fp == nullptr) return cudaErrorNotSupported;
  EncodeTiled enc = reinterpret_cast<EncodeTiled>(fp);
  cudaError_t err = cudaSuccess;
  if (prepared == nullptr) {
    err = launch_split_router(Wr, E, d, planes, stream);
    if (err != cudaSuccess) return err;
  } else {
    planes = const_cast<__nv_bfloat16*>(prepared);
  }
  CUtensorMap tx, tw;
  const cuuint64_t xdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
  const cuuint64_t wdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(RN)};
  const cuuint64_t stride[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t xbox[2] = {RK, RM};
  const cuuint32_t wbox[2] = {RK, RN / 2};
  const cuuint32_t es[2] = {1, 1};
  if (enc(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), xdim, stride, xbox, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, planes, wdim, stride, wbox, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(RSmem) + 1024;
  err = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  // One SM pair per 256 tokens (the last pair's odd CTA may hold none: its
  // token rows are read as zeros and nothing of it is stored).
  const int grid = 2 * ((T + 2 * RM - 1) / (2 * RM));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kRThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  note_launch();
  return cudaLaunchKernelEx(&cfg, router_tc_kernel, tx, tw, br, T, d, E, k, scale, idx, w, tile_counts, sb,
                            partitions == 2 ? 2 : 1);
}

}  // namespace mova
