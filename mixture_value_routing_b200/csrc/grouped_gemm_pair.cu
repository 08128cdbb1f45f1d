// Grouped expert GEMM on an SM pair (tcgen05 cta_group::2), bf16 -> fp32.
//
// Same computation as grouped_gemm_tc.cu -- for every pair p routed to
// expert e, P[p, r] = SiLU(Wv[e, r, :] . x[t(p), :]) ("MoVA: routing the
// value vectors, and why the KV cache does not notice", section "Where the
// routing happens"; the combine weights and sums the slots) -- with the MMA's
// M side spread over a cluster of two CTAs on neighbouring SMs:
//
//   * a tile is 256 weight rows x up to 256 pairs of one expert; the even CTA
//     holds weight rows 0..127 and the first half of the pairs, the odd CTA
//     rows 128..255 and the second half; one tcgen05.mma.cta_group::2 (M =
//     256, N <= 256, K = 16) reads both CTAs' shared memory and accumulates
//     into both CTAs' tensor memory (each its own 128 rows).
//   * Each CTA therefore loads per 64-wide K step only 16 KB of weights and
//     16 KB of token rows (vs 16 + 32 KB for one CTA doing half the work), and
//     the token tile is read n/256 instead of n/128 times.  Six 32 KB stages.
//   * Each CTA's TMA warp loads its own halves with 2-D tensor-map loads (no
//     multicast); completion is counted on the even CTA's stage barrier, for
//     which the even CTA alone declares the byte count of both halves.
//   * The even CTA's MMA thread issues the MMAs; tcgen05.commit with a
//     two-CTA multicast frees the stage in both CTAs and hands both
//     accumulators to the epilogues.  The odd CTA's epilogue releases an
//     accumulator with a remote arrive on the even CTA's barrier.
//   * Warps: 0 TMA, 1 MMA (even CTA), 2-5 epilogue (SiLU, bf16, store; rows
//     beyond the expert's n are skipped).  The epilogue reads the whole
//     accumulator into registers (bf16 pairs) and hands it back before it
//     stores, so the MMA of the tile after next never waits for the stores.
//   * One persistent pair per two SMs takes tiles from a global counter as
//     it goes (the even CTA's producer fetches the id and publishes it to
//     every role of both CTAs through a ring of mbarrier-guarded slots), so
//     unequal tile sizes do not leave some pairs a whole tile behind.  Tile
//     ids run expert by expert with the 4 weight-row tiles of a token tile
//     adjacent, so pairs working at the same time share the token rows in L2.
// Every mbarrier wait is bounded (MOVA_ERR_TIMEOUT); both CTAs meet at a
// cluster barrier before tensor memory is freed.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mova {

namespace {

constexpr int PM = 128;          // weight rows per CTA (256 per pair)
constexpr int PN = 256;          // pairs per tile
constexpr int PK = 64;
constexpr int kPStages = 6;
// Tile ids handed out dynamically pass through a ring in both CTAs'
// shared memory.  A role can lag the leader's producer by at most 8 tiles:
// the producer leads the MMA by at most kPStages k-steps (so at most 6
// tiles), the MMA leads the epilogues by the 2 accumulators.
constexpr int kTileRing = 16;
constexpr int kPABytes = PM * PK * 2;
constexpr int kPBBytes = (PN / 2) * PK * 2;
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPBoxRows = 32;
constexpr int kPThreads = 6 * 32;
constexpr uint32_t kPTmemCols = 512;

struct __align__(1024) PSmem {
  uint8_t stage[kPStages][kPStageBytes];
  uint64_t full[kPStages];   // even CTA: both halves of the stage landed
  uint64_t empty[kPStages];  // both CTAs: the pair's MMAs on the stage are done
  uint64_t tmem_full[2];     // both CTAs
  uint64_t tmem_empty[2];    // even CTA: 4 epilogue warps x 2 CTAs
  uint64_t tq_full[kTileRing];  // both CTAs: tile id i of this cluster published
  int tq[kTileRing];
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

struct PTile {
  int e, mt, tok0, valid, N, off;
};

__device__ __forceinline__ PTile decode_ptile(const PSmem& S, int t, int mtiles) {
  int a = 0;
  while (a + 1 < S.nact && S.tile_base[a + 1] <= t) ++a;
  const int local = t - S.tile_base[a];
  const int tt = local / mtiles;
  const int cnt = S.act_cnt[a];
  const int ntt = S.act_ntt[a];
  PTile r;
  r.e = S.act_e[a];
  r.mt = local - tt * mtiles;
  r.tok0 = static_cast<int>(static_cast<long long>(tt) * cnt / ntt);
  r.valid = static_cast<int>(static_cast<long long>(tt + 1) * cnt / ntt) - r.tok0;
  r.N = (r.valid + 15) & ~15;
  r.off = S.act_off[a];
  return r;
}

// The cluster's i-th tile id (waits until the even CTA's producer has
// published it; ntiles or more means no more tiles).  -1 if the wait ran out.
__device__ __forceinline__ int next_tile(PSmem& S, int i) {
  const int slot = i % kTileRing;
  if (!mbar_wait(&S.tq_full[slot], (i / kTileRing) & 1)) return -1;
  return *reinterpret_cast<volatile int*>(&S.tq[slot]);
}

__device__ __forceinline__ bool p_aborted(const PSmem& S) {
  return *reinterpret_cast<const volatile int*>(&S.abort) != 0;
}
__device__ __forceinline__ void p_fail(PSmem& S, StatusBlock* sb) {
  raise_status(sb, MOVA_ERR_TIMEOUT, static_cast<int32_t>(blockIdx.x));
  *reinterpret_cast<volatile int*>(&S.abort) = 1;
}

__global__ void __launch_bounds__(kPThreads, 1)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_xp,
                         const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                         const int32_t* __restrict__ active, StatusBlock* __restrict__ sb, int d, int n,
                         __nv_bfloat16* __restrict__ P) {
  extern __shared__ uint8_t smem_raw[];
  PSmem& S = *reinterpret_cast<PSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int mtiles = (n + 2 * PM - 1) / (2 * PM);
  const int nk = d / PK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.tmem_full[i], 1);
      mbar_init(&S.tmem_empty[i], 8);
    }
    for (int i = 0; i < kTileRing; ++i) mbar_init(&S.tq_full[i], 1);
    S.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, kPTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();  // grouping and gathered rows of this call are complete and visible
  if (threadIdx.x < 32) {
    const int nact = sb->num_active;
    int ntt0 = 0, ntt1 = 0;
    const int a0 = lane, a1 = lane + 32;
    if (a0 < nact) {
      const int e = active[a0];
      const int c = counts[e];
      S.act_e[a0] = e; S.act_cnt[a0] = c; S.act_off[a0] = offsets[e];
      ntt0 = (c + PN - 1) / PN;
      S.act_ntt[a0] = ntt0;
    }
    if (a1 < nact) {
      const int e = active[a1];
      const int c = counts[e];
      S.act_e[a1] = e; S.act_cnt[a1] = c; S.act_off[a1] = offsets[e];
      ntt1 = (c + PN - 1) / PN;
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
    if (lane == 31) S.ntiles = tot0 + v1;
  }
  tc_fence_before();
  cluster_sync_all();  // barriers and tensor memory of both CTAs are ready
  tc_fence_after();
  pdl_trigger();
  const int ntiles = S.ntiles;

  if (warp == 0) {
    // The whole warp runs the loop (warp-uniform state); one elected lane
    // issues the copies.  Stage and barrier addresses are computed once.
    // Tiles are handed out one at a time from a counter (zeroed by the
    // grouping of this call), so the clusters finish together however the
    // tile sizes fall.  The even CTA's producer takes each id and publishes it
    // to both CTAs; it requests the following id while it loads a tile.
    const uint32_t full0_cl = mapa_shared(smem_u32(&S.full[0]), 0);  // even CTA's barriers
    int s = 0;
    uint32_t phase = 0;
    bool started = false;
    int next = 0;
    if (rank == 0) {
      if (lane == 0) next = atomicAdd(&sb->work_next, 1);
      next = __shfl_sync(0xffffffffu, next, 0);
    }
    for (int i = 0;; ++i) {
      int t;
      if (rank == 0) {
        t = p_aborted(S) ? ntiles : next;
        if (elect_one()) {
          const int slot = i % kTileRing;
          S.tq[slot] = t;
          st_cluster_u32(mapa_shared(smem_u32(&S.tq[slot]), 1), static_cast<uint32_t>(t));
          mbar_arrive_cluster(mapa_shared(smem_u32(&S.tq_full[slot]), 1));
          mbar_arrive(&S.tq_full[slot]);
        }
        __syncwarp();
        if (t >= ntiles) break;
        if (lane == 0) next = atomicAdd(&sb->work_next, 1);  // read back at the next tile
        next = __shfl_sync(0xffffffffu, next, 0);
      } else {
        t = next_tile(S, i);
        if (t < 0) {
          if (lane == 0) p_fail(S, sb);
          break;
        }
        if (t >= ntiles) break;
      }
      const PTile tl = decode_ptile(S, t, mtiles);
      const int arow = tl.e * n + tl.mt * 2 * PM + static_cast<int>(rank) * PM;
      const int half = tl.N / 2;
      const int brow = tl.off + tl.tok0 + static_cast<int>(rank) * half;
      const int nbox = (half + kPBoxRows - 1) / kPBoxRows;
      const uint32_t bytes = 2u * static_cast<uint32_t>(kPABytes + nbox * kPBoxRows * PK * 2);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        // Slot s was used before (from the second pass over the ring on):
        // wait until the MMAs reading it have completed.
        if (started && !__all_sync(0xffffffffu, mbar_wait(&S.empty[s], phase ^ 1))) {
          if (lane == 0) p_fail(S, sb);
          ok = false;
          break;
        }
        if (elect_one()) {
          const uint32_t full_cl = full0_cl + static_cast<uint32_t>(s) * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&S.full[s], bytes);
          uint8_t* st = S.stage[s];
          tma_load_2d_pair(st, &tmap_w, kb * PK, arow, full_cl);
          for (int b = 0; b < nbox; ++b)
            tma_load_2d_pair(st + kPABytes + b * kPBoxRows * 128, &tmap_xp, kb * PK, brow + b * kPBoxRows, full_cl);
        }
        __syncwarp();
        if (++s == kPStages) {
          s = 0;
          phase ^= 1;
          started = true;
        }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // The whole warp runs the loop (so its state stays warp-uniform); one
      // elected lane issues the MMAs and commits.  Stage descriptors are
      // built once and advanced by adding offsets (start address in 16-byte
      // units), which keeps the issue cost below the MMA time even at
      // N = 144.
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(S.stage[0]));
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(S.stage[0]) + kPABytes);
      constexpr uint32_t kStageDesc = kPStageBytes >> 4;
      int s = 0;
      uint32_t phase = 0;
      for (int titer = 0;; ++titer) {
        const int t = next_tile(S, titer);
        if (t < 0) {
          if (lane == 0) p_fail(S, sb);
          break;
        }
        if (t >= ntiles || p_aborted(S)) break;
        const PTile tl = decode_ptile(S, t, mtiles);
        const int acc = titer & 1;
        if (titer >= 2 && !__all_sync(0xffffffffu, mbar_wait(&S.tmem_empty[acc], ((titer / 2) - 1) & 1))) {
          if (lane == 0) p_fail(S, sb);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = S.tmem_base + static_cast<uint32_t>(acc * PN);
        const uint32_t idesc = idesc_bf16_f32(2 * PM, tl.N);
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (!__all_sync(0xffffffffu, mbar_wait(&S.full[s], phase))) {
            if (lane == 0) p_fail(S, sb);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = adesc0 + static_cast<uint64_t>(s) * kStageDesc;
          const uint64_t db = bdesc0 + static_cast<uint64_t>(s) * kStageDesc;
          if (elect_one()) {
#pragma unroll
            for (int k16 = 0; k16 < PK / 16; ++k16)
              tc_mma_bf16_pair(d_tmem, da + 2 * k16, db + 2 * k16, idesc, (kb | k16) != 0);
            tc_commit_pair_both(&S.empty[s]);
          }
          __syncwarp();
          if (++s == kPStages) {
            s = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) tc_commit_pair_both(&S.tmem_full[acc]);
        __syncwarp();
      }
    }
  } else {
    const int lg = warp & 3;  // this warp may access TMEM lanes 32*lg .. 32*lg+31
    const uint32_t empty0 = mapa_shared(smem_u32(&S.tmem_empty[0]), 0);
    const uint32_t empty1 = mapa_shared(smem_u32(&S.tmem_empty[1]), 0);
    int titer = 0;
    for (;; ++titer) {
      const int t = next_tile(S, titer);
      if (t < 0) { p_fail(S, sb); break; }
      if (t >= ntiles || p_aborted(S)) break;
      const PTile tl = decode_ptile(S, t, mtiles);
      const int acc = titer & 1;
      if (!mbar_wait(&S.tmem_full[acc], (titer / 2) & 1)) { p_fail(S, sb); break; }
      tc_fence_after();
      const int rloc = tl.mt * 2 * PM + static_cast<int>(rank) * PM + lg * 32 + lane;
      const uint32_t tbase = S.tmem_base + static_cast<uint32_t>(acc * PN) +
                             (static_cast<uint32_t>(lg * 32) << 16);
      unsigned short* prow =
          reinterpret_cast<unsigned short*>(P + static_cast<size_t>(tl.off + tl.tok0) * n + rloc);
      const bool live = rloc < n;
      // All of the tile's columns go to registers first (SiLU, rounded to
      // bf16, two per word), so the accumulator is handed back to the MMA
      // before the stores start.
      uint32_t pk[PN / 32][16];
#pragma unroll
      for (int c = 0; c < PN / 32; ++c) {
        if (c * 32 < tl.N) {
          uint32_t r[32];
          tmem_ld_32(tbase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(silu_fast(__uint_as_float(r[2 * j])),
                                                           silu_fast(__uint_as_float(r[2 * j + 1])));
            pk[c][j] = *reinterpret_cast<const uint32_t*>(&h);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc == 0 ? empty0 : empty1);
      if (live) {
#pragma unroll
        for (int c = 0; c < PN / 32; ++c) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = c * 32 + j;
            if (col < tl.valid) {
              const uint32_t wv = pk[c][j >> 1];
              prow[static_cast<size_t>(col) * n] = static_cast<unsigned short>((j & 1) ? (wv >> 16) : (wv & 0xFFFFu));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while the pair may still touch its memory
  if (S.abort && threadIdx.x == 0) {
    for (int s = 0; s < kPStages; ++s) mbar_wait(&S.empty[s], 0);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(S.tmem_base, kPTmemCols);
  }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

}  // namespace

cudaError_t launch_tensor_experts_pair(const void* Wv, const int32_t* counts, const int32_t* offsets,
                                       const int32_t* active, StatusBlock* sb, int T, int d, int n,
                                       int k, int E, const __nv_bfloat16* xp, __nv_bfloat16* P,
                                       cudaStream_t stream) {
  void* fp = encode_tiled_fn();
  if (fp == nullptr) return cudaErrorNotSupported;
  EncodeTiled enc = reinterpret_cast<EncodeTiled>(fp);
  const int N = T * k;
  CUtensorMap tmap_w, tmap_xp;
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(E) * n};
  const cuuint64_t xdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {PK, PM};
  const cuuint32_t xbox[2] = {PK, kPBoxRows};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Wv), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&tmap_xp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(xp), xdim, gstride,
          xbox, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(PSmem) + 1024;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_pair_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  // As many pairs as can be resident at once (persistent).
  static int max_clusters = 0;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kPThreads);
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
  if (max_clusters == 0) {
    cfg.gridDim = dim3(2 * (sm_count() / 2));
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, grouped_gemm_pair_kernel, &cfg) != cudaSuccess || c <= 0)
      c = sm_count() / 2;
    max_clusters = c;
  }
  cfg.gridDim = dim3(2 * max_clusters);
  return cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel, tmap_w, tmap_xp, counts, offsets, active, sb,
                            d, n, P);
}

}  // namespace mova
