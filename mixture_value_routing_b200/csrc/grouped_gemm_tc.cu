// Grouped expert GEMM on 5th-generation tensor cores (tcgen05), bf16 -> fp32.
//
// For every active expert e and every (token, slot) pair p routed to it:
//   P[p, r] = SiLU( sum_j Wv[e, r, j] * x[t(p), j] )
// i.e. the k selected value projections of "MoVA: routing the value vectors,
// and why the KV cache does not notice" (section "Where the routing happens"),
// each passed through SiLU; the combine kernel weights them by their
// renormalised scores and sums the slots in fixed order.
//
// Tiles ("swap AB"): the MMA's M side is 128 weight rows of one expert, its N
// side up to 256 of the expert's pairs (ragged: rounded up to 16), K runs
// over d in 64-element steps.  An expert with c pairs is cut into ceil(c/256)
// near-equal token tiles, each combined with the n/128 weight-row tiles, so
// tail waste is below 16 columns per tile.
//
// First, gather_pairs_kernel copies each pair's x row into grouped order
// (xp[pos of pair (t, j)] = x[t], token-major), one bandwidth-bound pass, so that every
// token tile of the GEMM is a run of consecutive rows that TMA loads as
// plain 2-D boxes (token rows are read n/128 times, from L2, by TMA instead
// of 16-byte gathers through the load/store units).
//
// Then one persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: per 64-wide K step the weight tile (128 rows) and
//               the token tile (up to 256 rows of xp, in boxes of 32 rows),
//               both with 128-byte swizzle, completing on the stage mbarrier;
//   warp 1      MMA issuer (one thread): 4 x tcgen05.mma (K = 16) per stage
//               into a tensor-memory accumulator; tcgen05.commit frees the
//               stage and, per tile, hands the accumulator to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes, SiLU, bf16
//               round, store.
// Shared memory holds 4 stages of 48 KB; tensor memory holds two 256-column
// fp32 accumulators, so the epilogue of one tile overlaps the MMAs of the
// next.  Tiles are dealt round-robin over the CTAs in (expert, token tile,
// weight-row tile) order, so concurrently running CTAs share weight and x
// tiles in L2.  Every wait is bounded; a wait that runs out sets
// MOVA_ERR_TIMEOUT, every role leaves its loop, in-flight copies are drained
// and tensor memory is freed before the CTA exits.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mova {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int kStages = 4;
constexpr int kABytes = BM * BK * 2;
constexpr int kBBytes = BN * BK * 2;
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kBoxRows = 32;  // token rows per TMA box
constexpr int kWarpTma = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpEpi0 = 2;
constexpr int kEpiThreads = 128;
constexpr int kThreads = 6 * 32;
constexpr uint32_t kTmemCols = 512;

struct __align__(1024) Smem {
  uint8_t stage[kStages][kStageBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint32_t tmem_base;
  int abort;
  int ntiles;
  int nact;
  int act_e[64];
  int act_cnt[64];
  int act_off[64];
  int act_ntt[64];
  int tile_base[65];
};

struct Tile {
  int e, mt, tok0, valid, N, off;
};

__device__ __forceinline__ Tile decode_tile(const Smem& S, int t, int mtiles) {
  int a = 0;
  while (a + 1 < S.nact && S.tile_base[a + 1] <= t) ++a;
  const int local = t - S.tile_base[a];
  const int tt = local / mtiles;
  const int cnt = S.act_cnt[a];
  const int ntt = S.act_ntt[a];
  Tile r;
  r.e = S.act_e[a];
  r.mt = local - tt * mtiles;
  r.tok0 = static_cast<int>(static_cast<long long>(tt) * cnt / ntt);
  r.valid = static_cast<int>(static_cast<long long>(tt + 1) * cnt / ntt) - r.tok0;
  r.N = (r.valid + 15) & ~15;
  r.off = S.act_off[a];
  return r;
}

__device__ __forceinline__ bool aborted(const Smem& S) {
  return *reinterpret_cast<const volatile int*>(&S.abort) != 0;
}

__device__ __forceinline__ void fail(Smem& S, StatusBlock* sb) {
  raise_status(sb, MOVA_ERR_TIMEOUT, static_cast<int32_t>(blockIdx.x));
  *reinterpret_cast<volatile int*>(&S.abort) = 1;
}

__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_xp,
                    const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                    const int32_t* __restrict__ active, StatusBlock* __restrict__ sb, int d,
                    int n, int ldw, __nv_bfloat16* __restrict__ P) {
  extern __shared__ uint8_t smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mtiles = n / BM;
  const int nk = d / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.full[s], 1);                    // TMA arrive.expect_tx
      mbar_init(&S.empty[s], 1);                   // tcgen05.commit of the MMA thread
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.tmem_full[i], 1);
      mbar_init(&S.tmem_empty[i], kEpiThreads / 32);
    }
    S.abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // grouping and gathered rows of this call are complete and visible
  if (threadIdx.x < 32) {
    // Active experts, their pair counts and token-tile counts; tile prefix.
    const int nact = sb->num_active;
    int ntt0 = 0, ntt1 = 0;
    const int a0 = lane, a1 = lane + 32;
    if (a0 < nact) {
      const int e = active[a0];
      const int c = counts[e];
      S.act_e[a0] = e; S.act_cnt[a0] = c; S.act_off[a0] = offsets[e];
      ntt0 = (c + BN - 1) / BN;
      S.act_ntt[a0] = ntt0;
    }
    if (a1 < nact) {
      const int e = active[a1];
      const int c = counts[e];
      S.act_e[a1] = e; S.act_cnt[a1] = c; S.act_off[a1] = offsets[e];
      ntt1 = (c + BN - 1) / BN;
      S.act_ntt[a1] = ntt1;
    }
    int v0 = ntt0 * mtiles, v1 = ntt1 * mtiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, v0, o);
      const int y1 = __shfl_up_sync(0xffffffffu, v1, o);
      if (lane >= o) { v0 += y0; v1 += y1; }
    }
    const int tot0 = __shfl_sync(0xffffffffu, v0, 31);
    S.tile_base[a0 + 1] = v0;
    S.tile_base[a1 + 1] = tot0 + v1;
    if (lane == 0) {
      S.tile_base[0] = 0;
      S.nact = nact;
    }
    if (lane == 31) S.ntiles = tot0 + v1;  // tiles beyond nact contribute 0
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const int ntiles = S.ntiles;

  if (warp == kWarpTma) {
    if (lane == 0) {
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && !aborted(S); t += gridDim.x) {
        const Tile tl = decode_tile(S, t, mtiles);
        const int row = tl.e * ldw + tl.mt * BM;
        const int nbox = (tl.N + kBoxRows - 1) / kBoxRows;
        const uint32_t bytes = kABytes + nbox * kBoxRows * BK * 2;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(&S.empty[s], ((it / kStages) - 1) & 1)) { fail(S, sb); break; }
          mbar_arrive_expect_tx(&S.full[s], bytes);
          tma_load_2d_nohint(S.stage[s], &tmap_w, kb * BK, row, &S.full[s]);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_nohint(S.stage[s] + kABytes + b * kBoxRows * 128, &tmap_xp, kb * BK,
                               tl.off + tl.tok0 + b * kBoxRows, &S.full[s]);
        }
      }
    }
  } else if (warp == kWarpMma) {
    if (lane == 0) {
      int it = 0, titer = 0;
      for (int t = blockIdx.x; t < ntiles && !aborted(S); t += gridDim.x, ++titer) {
        const Tile tl = decode_tile(S, t, mtiles);
        const int acc = titer & 1;
        if (titer >= 2 && !mbar_wait(&S.tmem_empty[acc], ((titer / 2) - 1) & 1)) { fail(S, sb); break; }
        tc_fence_after();
        const uint32_t d_tmem = S.tmem_base + static_cast<uint32_t>(acc * BN);
        const uint32_t idesc = idesc_bf16_f32(BM, tl.N);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&S.full[s], (it / kStages) & 1)) { fail(S, sb); ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(S.stage[s]);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int k16 = 0; k16 < BK / 16; ++k16)
            tc_mma_bf16(d_tmem, smem_desc_sw128(a0 + k16 * 32), smem_desc_sw128(b0 + k16 * 32), idesc,
                        (kb | k16) != 0);
          tc_commit(&S.empty[s]);
        }
        if (!ok) break;
        tc_commit(&S.tmem_full[acc]);
      }
    }
  } else if (warp >= kWarpEpi0) {
    // No block-level barrier in this role, so a warp that gives up on a wait
    // can never leave the others stuck.  Thread = one weight row; columns =
    // the tile's pairs.
    const int lg = warp & 3;  // this warp may access TMEM lanes 32*lg .. 32*lg+31
    int titer = 0;
    for (int t = blockIdx.x; t < ntiles && !aborted(S); t += gridDim.x, ++titer) {
      const Tile tl = decode_tile(S, t, mtiles);
      const int acc = titer & 1;
      if (!mbar_wait(&S.tmem_full[acc], (titer / 2) & 1)) { fail(S, sb); break; }
      tc_fence_after();
      const int row = tl.mt * BM + lg * 32 + lane;
      const uint32_t tbase = S.tmem_base + static_cast<uint32_t>(acc * BN) +
                             (static_cast<uint32_t>(lg * 32) << 16);
      __nv_bfloat16* prow = P + static_cast<size_t>(tl.off + tl.tok0) * n + row;
      for (int c0 = 0; c0 < tl.N; c0 += 32) {
        uint32_t r[32];
        tmem_ld_32(tbase + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (c0 + j < tl.valid)
            prow[static_cast<size_t>(c0 + j) * n] = __float2bfloat16_rn(silu_fast(__uint_as_float(r[j])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.tmem_empty[acc]);
    }
  }

  __syncthreads();
  if (S.abort) {
    // Let every copy and MMA this CTA issued finish before its shared and
    // tensor memory are released (bounded: a dead wait just gives up).
    if (threadIdx.x == 0) {
      for (int s = 0; s < kStages; ++s) {
        mbar_wait(&S.full[s], 0);
        mbar_wait(&S.empty[s], 0);
      }
    }
    __syncthreads();
  }
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(S.tmem_base, kTmemCols);
  }
}

// xp[pos[t * k + j], :] = x[t, :] for every token t and slot j: one warp
// per token reads its row once (16-byte vectors, up to 8 per lane at a
// time) and writes it to the token's k grouped positions.  Token-major, so
// x is read once however large it is (in pair order each row would be read
// k times, from DRAM once x outgrows L2).  HBM-bound copy.
__global__ void __launch_bounds__(256)
gather_pairs_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ pos, int k, int vec_per_row,
                    int T, uint4* __restrict__ xp) {
  pdl_wait();
  // Evict-last: the rows are read again by the GEMM right after (once per
  // 256-row weight block), while the weights stream through L2 evict-first.
  // The same workspace rows are rewritten by every call.
  const uint64_t pol = policy_evict_last();
  const int lane = threadIdx.x & 31;
  const long long gw = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const long long nw = (static_cast<long long>(gridDim.x) * 256) >> 5;
  for (long long t = gw; t < T; t += nw) {
    const uint4* src = x + static_cast<size_t>(t) * vec_per_row;
    int p = 0;
    if (lane < k) p = pos[static_cast<size_t>(t) * k + lane];
    for (int v0 = 0; v0 < vec_per_row; v0 += 32 * 8) {
      uint4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int v = v0 + i * 32 + lane;
        if (v < vec_per_row) q[i] = src[v];
      }
      for (int j = 0; j < k; ++j) {
        uint4* dst = xp + static_cast<size_t>(__shfl_sync(0xffffffffu, p, j)) * vec_per_row;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int v = v0 + i * 32 + lane;
          if (v < vec_per_row)
            asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(dst + v),
                         "r"(q[i].x), "r"(q[i].y), "r"(q[i].z), "r"(q[i].w), "l"(pol)
                         : "memory");
        }
      }
    }
  }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

size_t tensor_experts_smem() { return sizeof(Smem) + 1024; }

cudaError_t launch_gather_pairs(const void* x, const int32_t* pos, int T, int d, int k,
                                __nv_bfloat16* xp, cudaStream_t stream) {
  const int vec_per_row = d / 8;
  long long blocks = (static_cast<long long>(T) * 32 + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  return launch_pdl(gather_pairs_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                    static_cast<const uint4*>(x), pos, k, vec_per_row, T, reinterpret_cast<uint4*>(xp));
}

cudaError_t launch_tensor_experts(const void* x, const void* Wv, long long ldw, const int32_t* counts,
                                  const int32_t* offsets, const int32_t* pos, const float* w32,
                                  const int32_t* active, StatusBlock* sb, int T, int d, int n, int k,
                                  int E, __nv_bfloat16* xp, __nv_bfloat16* P, cudaStream_t stream) {
  (void)w32;
  void* fp = encode_tiled_fn();
  if (fp == nullptr) return cudaErrorNotSupported;
  EncodeTiled enc = reinterpret_cast<EncodeTiled>(fp);
  const int N = T * k;
  // Rows of x in grouped order.
  cudaError_t err = launch_gather_pairs(x, pos, T, d, k, xp, stream);
  if (err != cudaSuccess) return err;
  // The experts as one (E*n) x d row-major bf16 matrix; boxes of 128 rows x
  // 64 columns (128 bytes) with 128-byte swizzle.  The gathered rows: N x d,
  // boxes of 32 rows.
  CUtensorMap tmap_w, tmap_xp;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d),
                              static_cast<cuuint64_t>(E - 1) * static_cast<cuuint64_t>(ldw) + n};
  const cuuint64_t xdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {BK, BM};
  const cuuint32_t xbox[2] = {BK, kBoxRows};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Wv), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&tmap_xp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, xp, xdim, gstride, xbox, estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = tensor_experts_smem();
  err = cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(grouped_gemm_kernel, dim3(sm_count()), dim3(kThreads), smem, stream, tmap_w, tmap_xp,
                    counts, offsets, active, sb, d, n, static_cast<int>(ldw), P);
}

}  // namespace mova
