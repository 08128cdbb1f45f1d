// Grouped expert GEMM on an SM pair (tcgen05 cta_group::2), bf16 -> fp32.
//
// For every pair p = (token t, slot) routed to expert e,
//   P[p, r] = SiLU(Wv[e, r, :] . x[t, :])
// ("MoVA: routing the value vectors, and why the KV cache does not notice",
// section "Where the routing happens": each selected expert's projection
// passes through SiLU; the combine weights it and sums the slots).  At
// prefill sizes this is a dense contraction -- 2 T k d n flop, 85.9 GFLOP
// at T = 4096 ("So what does it cost?": 10.49M multiply-accumulates per
// token) -- so it runs on the tensor cores:
//
//   * A tile is 256 weight rows of one expert (the MMA's M side, 128 rows in
//     each CTA of a two-CTA cluster) against up to 512 of that expert's
//     pairs (the N side, in two tensor-memory accumulators of up to 256
//     columns).  At ~256 pairs per expert every expert's weights are then
//     read once per 256-row block, and its pairs' token rows once per block.
//   * The token rows come from xp, the pairs' rows of x already gathered into
//     grouped order, so each CTA's share of a tile is two runs of consecutive
//     rows that 2-D TMA boxes of 32 rows load (TMA tile::gather4 straight from
//     x was measured at ~18 GB/s per SM, too slow to feed the MMA).
//   * Per 64-wide K step a CTA loads 16 KB of weights (one 2-D box) and up to
//     32 KB of token rows (its half of the tile's pairs: accumulator 0's rows
//     at the start of the stage's B area, accumulator 1's 16 KB further);
//     four 48 KB stages.  Batches of at most 256 pairs per expert on
//     average take tiles of up to 384 pairs instead (accumulator 1 at most
//     128), so a stage is 40 KB and five fit: more weight bytes in flight.
//     Both CTAs' copies complete on the even CTA's stage barrier (no
//     multicast).  The even CTA's MMA warp issues tcgen05.mma.cta_group::2
//     (M = 256, N = 16..256, K = 16) into accumulator 0 (pairs 0..255 of the
//     tile) and accumulator 1 (pairs 256..511); tcgen05.commit multicast
//     frees the stage in both CTAs.
//   * Tensor memory holds two 256-column accumulator regions.  A tile of at
//     most 256 pairs uses one, alternating, so its epilogue overlaps the next
//     tile's MMAs; a larger tile uses both.  Eight epilogue warps: four per
//     region, one per tensor-memory lane quarter.  Each reads the region's
//     columns into registers (SiLU, bf16) in two halves, storing the first
//     half before reading the second, and hands the region back right after
//     its last read; each 32 x 32 block goes through shared memory so that P
//     rows are stored as 16-byte vectors.
//   * Attend mode (the value side of decode attention over the compact
//     cache, V never stored): the epilogue instead sums, per weight row,
//     p[h, token] * w[pair] * SiLU(h) over the tile's pairs for the four
//     query heads of the CTA's KV head, and writes one partial per
//     token-tile group; attend_reduce_kernel adds them in a fixed order.
//   * One persistent pair per two SMs takes tiles from a global counter;
//     tiles are numbered largest expert first (then token tile, then the
//     four weight-row blocks of a token tile next to each other, so pairs
//     working at the same time share the token rows in L2), so the last
//     tiles handed out are the smallest.
// Every mbarrier wait is bounded (MOVA_ERR_TIMEOUT); on a failed wait every
// role leaves its loop, the copies and MMAs in flight are drained and tensor
// memory is freed.  Both CTAs meet at a cluster barrier before exiting.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mova {

namespace {

constexpr int PM = 128;         // weight rows per CTA (256 per pair)
constexpr int NA = 256;         // pairs per accumulator
constexpr int NT = 2 * NA;      // pairs per tile (the configuration of larger batches)
constexpr int NT_SMALL = NA + NA / 2;  // pairs per tile at <= 256 pairs per expert on average
constexpr int PK = 64;
constexpr int kTileRing = 16;
constexpr int kPABytes = PM * PK * 2;           // 16 KB of weights per stage
// The stage ring, in one of two configurations over the same shared-memory
// area: tiles of up to 512 pairs with four 48 KB stages (16 KB of weights and
// 32 KB of token rows per CTA), or tiles of up to 384 pairs with five 40 KB
// stages.  The second keeps more weight bytes in flight per SM; it is taken
// when the batch has at most 256 pairs per expert on average, where experts
// rarely need a second token tile (with 512-pair tiles fewer experts split,
// which matters at larger batches).
template <int kNT>
struct Ring {
  static constexpr int kStages = kNT > NT_SMALL ? 4 : 5;
  static constexpr int kBBytes = (kNT / 2) * PK * 2;
  static constexpr int kStageBytes = kPABytes + kBBytes;
};
constexpr int kPStagesMax = 5;
constexpr int kStageArea = Ring<NT_SMALL>::kStages * Ring<NT_SMALL>::kStageBytes;
static_assert(Ring<NT>::kStages * Ring<NT>::kStageBytes <= kStageArea, "both rings fit the stage area");
static_assert(Ring<NT_SMALL>::kStageBytes % 1024 == 0 && Ring<NT>::kStageBytes % 1024 == 0,
              "stages stay 1024-byte aligned (128-byte swizzle atoms)");
constexpr int kEpiWarps = 8;
constexpr int kPThreads = (2 + kEpiWarps) * 32;  // warp 0 TMA, warp 1 MMA, 2-9 epilogue
constexpr uint32_t kPTmemCols = 512;

struct __align__(1024) PSmem {
  uint8_t stage_area[kStageArea];  // Ring<kNT>::kStages stages of Ring<kNT>::kStageBytes
  uint64_t full[kPStagesMax];   // even CTA: both CTAs' copies of the stage landed
  uint64_t empty[kPStagesMax];  // both CTAs: the pair's MMAs on the stage are done
  uint64_t reg_full[2];         // both CTAs: tensor-memory region r holds a finished accumulator
  uint64_t reg_empty[2];        // even CTA: region r read out by its 4 epilogue warps x 2 CTAs
  uint64_t tq_full[kTileRing];  // both CTAs: tile id i of this cluster published
  int tq[kTileRing];
  uint32_t tmem_base;
  int abort;
  int ntiles;
  int nact;
  // Active experts in tile order (largest pair count first).
  int act_e[64];
  int act_cnt[64];
  int act_off[64];
  int act_ntt[64];
  int act_gbase[64];  // attend mode: the expert's first token-tile group (experts in index order)
  int tile_base[65];
  // Per epilogue warp: a 32 x 32 bf16 block transposed for the P stores
  // (column-major, rows paired into 32-bit words).
  alignas(16) uint32_t epi[kEpiWarps][32 * 16];  // read as 16-byte vectors
};

struct PTile {
  int e, mt, tt, ntt, tok0, valid, N0, N1, off, gbase;
};

__device__ __forceinline__ PTile decode_ptile(const PSmem& S, int t, int mtiles) {
  // The expert of tile t: the last a with tile_base[a] <= t (tile_base is
  // strictly increasing over the active experts).
  int a = 0, hi = S.nact - 1;
  while (a < hi) {
    const int mid = (a + hi + 1) >> 1;
    if (S.tile_base[mid] <= t) a = mid; else hi = mid - 1;
  }
  const int local = t - S.tile_base[a];
  const int tt = local / mtiles;
  const int cnt = S.act_cnt[a];
  const int ntt = S.act_ntt[a];
  PTile r;
  r.e = S.act_e[a];
  r.tt = tt;
  r.ntt = ntt;
  r.gbase = S.act_gbase[a];
  r.mt = local - tt * mtiles;
  r.tok0 = static_cast<int>(static_cast<long long>(tt) * cnt / ntt);
  r.valid = static_cast<int>(static_cast<long long>(tt + 1) * cnt / ntt) - r.tok0;
  const int N = (r.valid + 15) & ~15;
  r.N0 = min(N, NA);
  r.N1 = N - r.N0;
  r.off = S.act_off[a];
  return r;
}

// Inclusive prefix over 64 values, v0 of lane l at index l and v1 at 32 + l;
// tot0 = sum of the first 32, tot = sum of all.
__device__ __forceinline__ void tile_prefix(int& v0, int& v1, int lane, int& tot0, int& tot) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(0xffffffffu, v0, o);
    const int y1 = __shfl_up_sync(0xffffffffu, v1, o);
    if (lane >= o) { v0 += y0; v1 += y1; }
  }
  tot0 = __shfl_sync(0xffffffffu, v0, 31);
  tot = tot0 + __shfl_sync(0xffffffffu, v1, 31);
}

// Attend mode (the PV product of decode attention with V recomputed from the
// compact cache, never stored): per query head h and cached position l,
// p[h * L + l] is the attention probability; query head h reads KV head
// h / G.  Each tile leaves, per query head of its KV head and weight row,
// the sum over its pairs of p[h, token] * w[pair] * SiLU(h_pair[row]) in
// part[((group * 2 + accumulator) * G + head-in-group) * n + row].
// coef[q * Hp + 4 * g + j] = p[(g * G + j) * L + token of pair q] * w[pair q]
// for grouped position q, KV head g and head-in-group j < G (zero for
// G <= j < 4): prepared by attend_coef_kernel.
struct AttendArgs {
  const float* coef;
  float* part;
  int Hp;  // 4 * KV heads
};

// Tensor memory holds two accumulator regions of 256 columns.  A tile of at
// most 256 pairs takes one region, alternating between the two, so its
// epilogue overlaps the next tile's MMAs; a larger tile takes both (pairs
// 0..255 in the next region, the rest in the other), and the tile after it
// starts in the region of that smaller second accumulator, which its
// epilogue hands back first.  Every role walks the cluster's tile sequence
// and applies this rule, so they agree on which region holds what, and on
// each region's use count (its barrier parity).
struct Regions {
  int next = 0;
  int uses0 = 0, uses1 = 0;
  __device__ __forceinline__ int uses(int r) const { return r == 0 ? uses0 : uses1; }
  __device__ __forceinline__ void used(int r) {
    if (r == 0) ++uses0; else ++uses1;
  }
  // Regions of a tile: r0 for its first accumulator, r1 for its second (-1
  // if none).
  __device__ __forceinline__ void take(const PTile& tl, int& r0, int& r1) {
    r0 = next;
    r1 = tl.N1 > 0 ? next ^ 1 : -1;
    next ^= 1;
  }
};

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

constexpr int kBoxRows = 32;                    // token rows per TMA box
constexpr int kAcc1Rows = NA / 2;               // accumulator 1's rows start here in B

// Ten warps: sub-partitions 0 and 1 hold three each, so at most
// 16384 / (3 * 32) -> 168 registers per thread.
template <bool kAttend, int kNT>
__global__ void __maxnreg__(168)
grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_xp,
                         const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                         int E, StatusBlock* __restrict__ sb, int d, int n,
                         int ldw, __nv_bfloat16* __restrict__ P, AttendArgs at) {
  extern __shared__ uint8_t smem_raw[];
  PSmem& S = *reinterpret_cast<PSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  using R = Ring<kNT>;
  static_assert(!kAttend || kNT == NT, "attend partials are laid out for 512-pair tiles");
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int mtiles = (n + 2 * PM - 1) / (2 * PM);
  const int nk = d / PK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < R::kStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.reg_full[i], 1);
      mbar_init(&S.reg_empty[i], 4 * 2);
    }
    for (int i = 0; i < kTileRing; ++i) mbar_init(&S.tq_full[i], 1);
    S.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&S.tmem_base, kPTmemCols);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the grouping of this call is complete and visible
  if (threadIdx.x < 32) {
    // The active experts (count > 0) ordered by pair count, descending
    // (equal counts keep ascending expert order), then the tile prefix.
    // Lane l holds experts l and l + 32; all four reads go out at once.
    const int e0 = lane, e1 = lane + 32;
    const int c0 = e0 < E ? counts[e0] : 0;
    const int c1 = e1 < E ? counts[e1] : 0;
    const int f0 = e0 < E ? offsets[e0] : 0;
    const int f1 = e1 < E ? offsets[e1] : 0;
    int r0 = 0, r1 = 0;  // experts ahead of e0 / e1 in that order
    for (int b = 0; b < 32; ++b) {
      const int x0 = __shfl_sync(0xffffffffu, c0, b);  // count of expert b
      const int x1 = __shfl_sync(0xffffffffu, c1, b);  // count of expert b + 32
      r0 += (x0 > c0 || (x0 == c0 && b < lane)) + (x1 > c0);
      r1 += (x0 >= c1) + (x1 > c1 || (x1 == c1 && b < lane));
    }
    const int nact = __popc(__ballot_sync(0xffffffffu, c0 > 0)) + __popc(__ballot_sync(0xffffffffu, c1 > 0));
    // Token-tile groups in expert index order (attend mode: one partial per
    // group, accumulator, query head of the group and weight row).
    int q0 = c0 > 0 ? (c0 + kNT - 1) / kNT : 0, q1 = c1 > 0 ? (c1 + kNT - 1) / kNT : 0;
    {
      int g0 = q0, g1 = q1, gt0, gt;
      tile_prefix(g0, g1, lane, gt0, gt);
      q0 = g0 - q0;        // exclusive: groups of experts below e0
      q1 = gt0 + g1 - q1;  // and below e1
    }
    if (c0 > 0) S.act_gbase[r0] = q0;
    if (c1 > 0) S.act_gbase[r1] = q1;
    if (c0 > 0) {
      S.act_e[r0] = e0;
      S.act_cnt[r0] = c0;
      S.act_off[r0] = f0;
      S.act_ntt[r0] = (c0 + kNT - 1) / kNT;
    }
    if (c1 > 0) {
      S.act_e[r1] = e1;
      S.act_cnt[r1] = c1;
      S.act_off[r1] = f1;
      S.act_ntt[r1] = (c1 + kNT - 1) / kNT;
    }
    __syncwarp();
    const int a0 = lane, a1 = lane + 32;
    int v0 = a0 < nact ? S.act_ntt[a0] * mtiles : 0;
    int v1 = a1 < nact ? S.act_ntt[a1] * mtiles : 0;
    int tot0, tot;
    tile_prefix(v0, v1, lane, tot0, tot);
    S.tile_base[a0 + 1] = v0;
    S.tile_base[a1 + 1] = tot0 + v1;
    if (lane == 0) {
      S.tile_base[0] = 0;
      S.nact = nact;
    }
    if (lane == 31) S.ntiles = tot0 + v1;
  }
  tc_fence_before();
  cluster_sync_all();  // barriers, expert order and tensor memory of both CTAs are ready
  tc_fence_after();
  pdl_trigger();
  const int ntiles = S.ntiles;

  if (warp == 0) {
    // The whole warp runs the loop (warp-uniform state); one elected lane
    // declares the stage's bytes and issues the copies.  The even CTA's
    // producer takes the tile ids from the global counter (zeroed by this
    // call's grouping) and publishes each to both CTAs.
    const uint32_t full0_cl = mapa_shared(smem_u32(&S.full[0]), 0);  // even CTA's barriers
    // A weight block read by one tile only (the expert has one token tile)
    // streams through evict-first, so the gathered token rows (stored
    // evict-last) stay in L2 for the four weight-row blocks that read them;
    // the blocks of experts with several token tiles keep the normal policy,
    // as those tiles read them about together.
    const uint64_t wpol = policy_evict_first();
    int s = 0;
    uint32_t phase = 0;
    bool started = false;
    // Cluster c takes tile c first, then ids ncl + (counter value).  Lane 0
    // fetches the next id one tile ahead, so the atomic's round trip never
    // holds up a tile's first copies.
    const int ncl = static_cast<int>(gridDim.x) / 2;
    int nraw = 0;
    if (rank == 0 && lane == 0) nraw = ncl + atomicAdd(&sb->work_next, 1);
    for (int i = 0;; ++i) {
      int t;
      if (rank == 0) {
        const int nxt = i == 0 ? static_cast<int>(blockIdx.x) / 2 : __shfl_sync(0xffffffffu, nraw, 0);
        t = p_aborted(S) ? ntiles : nxt;
        if (elect_one()) {
          const int slot = i % kTileRing;
          S.tq[slot] = t;
          st_cluster_u32(mapa_shared(smem_u32(&S.tq[slot]), 1), static_cast<uint32_t>(t));
          mbar_arrive_cluster(mapa_shared(smem_u32(&S.tq_full[slot]), 1));
          mbar_arrive(&S.tq_full[slot]);
        }
        __syncwarp();
        if (t >= ntiles) break;
        if (i > 0 && lane == 0) nraw = ncl + atomicAdd(&sb->work_next, 1);  // read at the next tile
      } else {
        t = next_tile(S, i);
        if (t < 0) {
          if (lane == 0) p_fail(S, sb);
          break;
        }
        if (t >= ntiles) break;
      }
      const PTile tl = decode_ptile(S, t, mtiles);
      const int arow = tl.e * ldw + tl.mt * 2 * PM + static_cast<int>(rank) * PM;
      // This CTA's B rows: the first half (rank 0) or second half (rank 1)
      // of accumulator 0's pairs, then likewise of accumulator 1's, each a
      // run of consecutive xp rows.  Boxes of 32 rows may read past a run's
      // end (rows of the next pairs, or zeros past the last pair): those rows
      // land inside the run's 16 KB of B and no MMA reads them.
      const int h0 = tl.N0 / 2, h1 = tl.N1 / 2;
      const int row0 = tl.off + tl.tok0 + static_cast<int>(rank) * h0;
      const int row1 = tl.off + tl.tok0 + tl.N0 + static_cast<int>(rank) * h1;
      const int nb0 = (h0 + kBoxRows - 1) / kBoxRows;
      const int nb1 = (h1 + kBoxRows - 1) / kBoxRows;
      const uint32_t bytes = 2u * static_cast<uint32_t>(kPABytes + (nb0 + nb1) * kBoxRows * PK * 2);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        // Slot s was used before (from the second pass over the ring on):
        // wait until the MMAs reading it have completed.
        if (started && !__all_sync(0xffffffffu, mbar_wait(&S.empty[s], phase ^ 1))) {
          if (lane == 0) p_fail(S, sb);
          ok = false;
          break;
        }
        const uint32_t full_cl = full0_cl + static_cast<uint32_t>(s) * 8u;
        uint8_t* st = S.stage_area + s * R::kStageBytes;
        if (elect_one()) {
          if (rank == 0) mbar_arrive_expect_tx(&S.full[s], bytes);
          if (tl.ntt == 1)
            tma_load_2d_pair_hint(st, &tmap_w, kb * PK, arow, full_cl, wpol);
          else  // the expert's other token tiles read this weight block too
            tma_load_2d_pair(st, &tmap_w, kb * PK, arow, full_cl);
          uint8_t* bt = st + kPABytes;
          for (int b = 0; b < nb0; ++b)
            tma_load_2d_pair(bt + b * kBoxRows * 128, &tmap_xp, kb * PK, row0 + b * kBoxRows, full_cl);
          for (int b = 0; b < nb1; ++b)
            tma_load_2d_pair(bt + (kAcc1Rows + b * kBoxRows) * 128, &tmap_xp, kb * PK, row1 + b * kBoxRows,
                             full_cl);
        }
        __syncwarp();
        if (++s == R::kStages) {
          s = 0;
          phase ^= 1;
          started = true;
        }
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    if (rank == 0) {
      // The whole warp runs the loop; one elected lane issues the MMAs and
      // commits.  Stage descriptors are built once and advanced by adding
      // offsets (start address in 16-byte units).
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(S.stage_area));
      const uint64_t bdesc0 = smem_desc_sw128(smem_u32(S.stage_area) + kPABytes);
      constexpr uint32_t kStageDesc = R::kStageBytes >> 4;
      int s = 0;
      uint32_t phase = 0;
      Regions reg;
      for (int titer = 0;; ++titer) {
        const int t = next_tile(S, titer);
        if (t < 0) {
          if (lane == 0) p_fail(S, sb);
          break;
        }
        if (t >= ntiles || p_aborted(S)) break;
        const PTile tl = decode_ptile(S, t, mtiles);
        int r0, r1;
        reg.take(tl, r0, r1);
        const uint32_t d0 = S.tmem_base + static_cast<uint32_t>(r0 * NA);
        const uint32_t d1 = S.tmem_base + static_cast<uint32_t>((r1 < 0 ? 0 : r1) * NA);
        const uint32_t idesc0 = idesc_bf16_f32(2 * PM, tl.N0);
        const uint32_t idesc1 = idesc_bf16_f32(2 * PM, tl.N1 > 0 ? tl.N1 : 16);
        // Accumulator 1's B rows start kAcc1Rows rows into each CTA's B area.
        const uint64_t b1off = static_cast<uint64_t>(kAcc1Rows * PK * 2) >> 4;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
          if (kb == 0) {
            // The regions this tile writes must have been read out by the
            // epilogues of their previous uses.
            bool got = true;
            if (reg.uses(r0) > 0) got = mbar_wait(&S.reg_empty[r0], (reg.uses(r0) - 1) & 1);
            if (got && r1 >= 0 && reg.uses(r1) > 0) got = mbar_wait(&S.reg_empty[r1], (reg.uses(r1) - 1) & 1);
            if (!__all_sync(0xffffffffu, got)) {
              if (lane == 0) p_fail(S, sb);
              ok = false;
              break;
            }
            tc_fence_after();
          }
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
              tc_mma_bf16_pair(d0, da + 2 * k16, db + 2 * k16, idesc0, (kb | k16) != 0);
            if (tl.N1 > 0) {
#pragma unroll
              for (int k16 = 0; k16 < PK / 16; ++k16)
                tc_mma_bf16_pair(d1, da + 2 * k16, db + b1off + 2 * k16, idesc1, (kb | k16) != 0);
            }
            tc_commit_pair_both(&S.empty[s]);
          }
          __syncwarp();
          if (++s == R::kStages) {
            s = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (elect_one()) {
          tc_commit_pair_both(&S.reg_full[r0]);
          if (r1 >= 0) tc_commit_pair_both(&S.reg_full[r1]);
        }
        __syncwarp();
        reg.used(r0);
        if (r1 >= 0) reg.used(r1);
      }
    }
  } else {
    // Epilogue: warp w reads tensor-memory lanes 32 * (w % 4) .. +31 (its
    // CTA's weight rows) of region (w - 2) / 4, for every tile that uses it.
    const int q = warp & 3;
    const int myreg = (warp - 2) / 4;
    const uint32_t empty_cl = mapa_shared(smem_u32(&S.reg_empty[myreg]), 0);
    Regions reg;
    for (int titer = 0;; ++titer) {
      const int t = next_tile(S, titer);
      if (t < 0) { p_fail(S, sb); break; }
      if (t >= ntiles || p_aborted(S)) break;
      const PTile tl = decode_ptile(S, t, mtiles);
      int r0, r1;
      reg.take(tl, r0, r1);
      if (myreg != r0 && myreg != r1) continue;  // this tile leaves the region alone
      const int acc = myreg == r0 ? 0 : 1;       // which of the tile's accumulators it holds
      if (!mbar_wait(&S.reg_full[myreg], reg.uses(myreg) & 1)) { p_fail(S, sb); break; }
      reg.used(myreg);
      tc_fence_after();
      const int N = acc == 0 ? tl.N0 : tl.N1;
      const int j0 = acc == 0 ? 0 : tl.N0;  // the tile's pair of this accumulator's column 0
      const int nvalid = min(N, tl.valid - j0);
      const int rloc = tl.mt * 2 * PM + static_cast<int>(rank) * PM + q * 32 + lane;
      const uint32_t tbase = S.tmem_base + static_cast<uint32_t>(myreg * NA) + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kAttend) {
        // Attend mode: the weighted sums of SiLU(h) over the unit's pairs
        // for the four query heads of this CTA's KV head, per weight row.
        const int rb = rloc - lane;             // this warp's first weight row
        const int head = (rloc - q * 32 - lane) / 128;  // the CTA's 128 rows are one KV head
        float4* cw = reinterpret_cast<float4*>(S.epi[warp - 2]);  // 32 columns' coefficients
        const float* cbase = at.coef + static_cast<size_t>(tl.off + tl.tok0 + j0) * at.Hp + 4 * head;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
        float4 cn = make_float4(0.f, 0.f, 0.f, 0.f);
        if (rb < n && lane < nvalid) cn = __ldg(reinterpret_cast<const float4*>(cbase + static_cast<size_t>(lane) * at.Hp));
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          if (cc * 32 >= N) break;
          const float4 c = cn;
          cn = make_float4(0.f, 0.f, 0.f, 0.f);
          const int nxt = (cc + 1) * 32 + lane;
          if (rb < n && nxt < nvalid && (cc + 1) * 32 < N)
            cn = __ldg(reinterpret_cast<const float4*>(cbase + static_cast<size_t>(nxt) * at.Hp));
          uint32_t r[32];
          tmem_ld_32(tbase + cc * 32, r);
          cw[lane] = c;
          tmem_ld_wait();
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float4 cj = cw[j];
            const float sv = silu_fast(__uint_as_float(r[j]));
            a0 = fmaf(cj.x, sv, a0);
            a1 = fmaf(cj.y, sv, a1);
            a2 = fmaf(cj.z, sv, a2);
            a3 = fmaf(cj.w, sv, a3);
          }
          __syncwarp();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(empty_cl);
        if (rb < n) {
          float* pp = at.part + static_cast<size_t>((tl.gbase + tl.tt) * 2 + acc) * 4 * n + rloc;
          pp[0] = a0;
          pp[static_cast<size_t>(n)] = a1;
          pp[2 * static_cast<size_t>(n)] = a2;
          pp[3 * static_cast<size_t>(n)] = a3;
          if (acc == 0 && tl.N1 == 0) {
            // No second accumulator: its slot of this group holds zeros.
#pragma unroll
            for (int j = 0; j < 4; ++j) pp[static_cast<size_t>(4 + j) * n] = 0.f;
          }
        }
        continue;
      }
      // The accumulator's columns are read in two halves of 128 (SiLU,
      // rounded to bf16, two per word): the first half is read and stored,
      // then the second half is read, the accumulator is handed back to the
      // MMA, and the second half is stored.  An accumulator of at most 128
      // columns is handed back right after its only read.  (Three of the ten warps share a
      // sub-partition's 16K registers, so a thread cannot hold all 256
      // columns at once.)
      // The warp's 32 weight rows are all below n or all at or above it (n
      // is a multiple of 128).  Lane l stores rows rbase + 8 (l % 4) ..
      // + 7 of a pair's P row as one 16-byte vector.
      const int rbase = rloc - lane;
      const bool live = rbase < n;
      uint32_t* Tw = S.epi[warp - 2];
      __nv_bfloat16* pseg = P + static_cast<size_t>(tl.off + tl.tok0 + j0) * n + rbase + (lane & 3) * 8;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pk[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int cc = 4 * h + c;
          if (cc * 32 < N) {
            uint32_t r[32];
            tmem_ld_32(tbase + cc * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const __nv_bfloat162 v2 = __floats2bfloat162_rn(silu_fast(__uint_as_float(r[2 * j])),
                                                              silu_fast(__uint_as_float(r[2 * j + 1])));
              pk[c][j] = *reinterpret_cast<const uint32_t*>(&v2);
            }
          }
        }
        if (h == (N > 128 ? 1 : 0)) {  // after the last read of the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(empty_cl);
        }
        if (live) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int cb = (4 * h + c) * 32;  // the block's first column (pair)
            if (cb < nvalid) {
              // Transpose the 32 rows x 32 columns block through shared
              // memory: lanes 2i and 2i + 1 pair their rows into one word
              // per column (even lane: column 2j, odd lane: column 2j + 1).
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const uint32_t mine = pk[c][j];
                const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                const uint32_t w = (lane & 1) ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
                Tw[(2 * j + (lane & 1)) * 16 + (lane >> 1)] = w;
              }
              __syncwarp();
#pragma unroll
              for (int it = 0; it < 4; ++it) {
                const int cc = it * 8 + (lane >> 2);
                if (cb + cc < nvalid)
                  *reinterpret_cast<uint4*>(pseg + static_cast<size_t>(cb + cc) * n) =
                      *reinterpret_cast<const uint4*>(&Tw[cc * 16 + (lane & 3) * 4]);
              }
              __syncwarp();
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while the pair may still touch its memory
  if (S.abort && threadIdx.x == 0) {
    for (int s = 0; s < R::kStages; ++s) mbar_wait(&S.empty[s], 0);
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

namespace {

template <bool kAttend, int kNT>
cudaError_t launch_pair(const void* Wv, long long ldw, const int32_t* counts, const int32_t* offsets,
                        StatusBlock* sb, int T, int d, int n, int k, int E, const __nv_bfloat16* xp,
                        __nv_bfloat16* P, AttendArgs at, cudaStream_t stream) {
  void* fp = encode_tiled_fn();
  if (fp == nullptr) return cudaErrorNotSupported;
  EncodeTiled enc = reinterpret_cast<EncodeTiled>(fp);
  CUtensorMap tmap_w, tmap_xp;
  // The experts' rows as one matrix: expert e's row r is row e * ldw + r;
  // rows between n and ldw (another rank's slice) are read by a weight tile
  // that runs past n but never stored.
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(d),
                              static_cast<cuuint64_t>(E - 1) * static_cast<cuuint64_t>(ldw) + n};
  const cuuint64_t xdim[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T) * k};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t box[2] = {PK, PM};
  const cuuint32_t xbox[2] = {PK, kBoxRows};
  const cuuint32_t estride[2] = {1, 1};
  if (enc(&tmap_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(Wv), gdim, gstride, box,
          estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&tmap_xp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(xp), xdim, gstride, xbox,
          estride,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(PSmem) + 1024;
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<kAttend, kNT>,
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
    if (cudaOccupancyMaxActiveClusters(&c, grouped_gemm_pair_kernel<kAttend, kNT>, &cfg) != cudaSuccess || c <= 0)
      c = sm_count() / 2;
    max_clusters = c;
  }
  cfg.gridDim = dim3(2 * max_clusters);
  note_launch();
  return cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<kAttend, kNT>, tmap_w, tmap_xp, counts, offsets, E, sb, d,
                            n, static_cast<int>(ldw), P, at);
}

// coef[q * Hp + 4 * g + j] for every grouped position q (see AttendArgs):
// one thread per (q, KV head g), four query heads each.
__global__ void __launch_bounds__(256)
attend_coef_kernel(const float* __restrict__ probs, const int32_t* __restrict__ perm,
                   const float* __restrict__ w32, int L, int k, int nkv, int G, float* __restrict__ coef) {
  pdl_wait();
  const long long total = static_cast<long long>(L) * k * nkv;
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * 256) {
    const int q = static_cast<int>(i / nkv);
    const int g = static_cast<int>(i % nkv);
    const int f = perm[q];
    const int pos = f / k;
    const float wq = w32[f];
    float c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      c[j] = j < G ? probs[static_cast<size_t>(g * G + j) * L + pos] * wq : 0.f;
    *reinterpret_cast<float4*>(coef + static_cast<size_t>(q) * 4 * nkv + 4 * g) =
        make_float4(c[0], c[1], c[2], c[3]);
  }
}

// o[h, c] = sum over token-tile groups (expert order, then token tile) and
// accumulators of part[((group * 2 + acc) * 4 + h % G) * n + (h / G) * 128 + c].
// A block of 32 warps takes query head h and 32 columns: warp w sums groups
// w, w + 32, ... (both accumulators, in group order), lane = column; warp 0
// then adds the 32 warps' sums in warp order.  A fixed order, so the result
// does not depend on timing.
__global__ void __launch_bounds__(1024)
attend_reduce_kernel(const float* __restrict__ part, const int32_t* __restrict__ counts, int E, int n,
                     int G, int H, float* __restrict__ o) {
  pdl_wait();
  __shared__ int ngroups;
  __shared__ float red[32][33];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    int g = 0;
    for (int e = 0; e < E; ++e) g += (counts[e] + NT - 1) / NT;
    ngroups = g;
  }
  __syncthreads();
  const int h = blockIdx.x / 4;
  const int c = (blockIdx.x % 4) * 32 + lane;
  const size_t col = static_cast<size_t>((h / G) * 128 + c);
  const size_t hq = static_cast<size_t>(h % G);
  float acc = 0.f;
  for (int g = warp; g < ngroups; g += 32) {
    acc += part[((static_cast<size_t>(g) * 2) * 4 + hq) * n + col];
    acc += part[((static_cast<size_t>(g) * 2 + 1) * 4 + hq) * n + col];
  }
  red[warp][lane] = acc;
  __syncthreads();
  if (warp == 0) {
    float t = 0.f;
    for (int w = 0; w < 32; ++w) t += red[w][lane];
    o[static_cast<size_t>(h) * 128 + c] = t;
  }
}

}  // namespace

cudaError_t launch_tensor_experts_pair(const void* Wv, long long ldw, const int32_t* counts,
                                       const int32_t* offsets, StatusBlock* sb, int T,
                                       int d, int n, int k, int E, const __nv_bfloat16* xp, __nv_bfloat16* P,
                                       cudaStream_t stream) {
  // At most 256 pairs per expert on average: the 384-pair tiles and the
  // deeper ring; otherwise the 512-pair tiles.
  if (static_cast<long long>(T) * k <= 256LL * E)
    return launch_pair<false, NT_SMALL>(Wv, ldw, counts, offsets, sb, T, d, n, k, E, xp, P, AttendArgs{}, stream);
  return launch_pair<false, NT>(Wv, ldw, counts, offsets, sb, T, d, n, k, E, xp, P, AttendArgs{}, stream);
}

size_t attend_part_bytes(int L, int E, int k, int n) {
  const long long groups = static_cast<long long>(L) * k / NT + E + 1;
  return static_cast<size_t>(groups) * 2 * 4 * n * 4;
}

cudaError_t launch_tensor_attend(const void* Wv, const int32_t* counts, const int32_t* offsets,
                                 const int32_t* perm, const float* w32, StatusBlock* sb, int L, int d, int n,
                                 int k, int E, const float* probs, int H, const __nv_bfloat16* xp,
                                 float* coef, float* part, float* o, cudaStream_t stream) {
  const int nkv = n / 128;
  const int G = H / nkv;
  const long long total = static_cast<long long>(L) * k * nkv;
  long long blocks = (total + 255) / 256;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaError_t err = launch_pdl(attend_coef_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                               probs, perm, w32, L, k, nkv, G, coef);
  if (err != cudaSuccess) return err;
  err = launch_pair<true, NT>(Wv, n, counts, offsets, sb, L, d, n, k, E, xp, nullptr,
                          AttendArgs{coef, part, 4 * nkv}, stream);
  if (err != cudaSuccess) return err;
  return launch_pdl(attend_reduce_kernel, dim3(static_cast<unsigned>(H * 4)), dim3(1024), 0, stream,
                    static_cast<const float*>(part), counts, E, n, G, H, o);
}

}  // namespace mova
