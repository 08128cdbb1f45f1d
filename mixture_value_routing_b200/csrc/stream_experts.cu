// Weight-streaming expert kernel for decode-sized batches (and the fp32 path).
//
// Computes, for every (token, slot) pair p routed to expert e,
//   P[p, :] = SiLU(Wv[e] x[t])
// as in "MoVA: routing the value vectors, and why the KV cache does not
// notice", section "Where the routing happens" (each selected expert's
// projection passes through SiLU; the combine weights it by its renormalised
// score and sums the slots).
//
// At a few tokens per expert this is a matrix-vector product per active
// expert and HBM-bound: each active expert's n x d weight is read exactly
// once, by one persistent CTA per SM.  In each CTA a producer warp streams
// 8-row slabs into a ring of 4 shared-memory stages with 1-D bulk (TMA)
// copies completing on mbarriers (lanes 0-7 issue a stage's eight row copies
// together), so each SM keeps ~160 KB of weights in flight without spending
// registers on it.  Eight consumer warps split K and run mma.sync m16n8k16
// on (8 weight rows) x (8 token columns).
//
// Decode batches (bf16, T <= 8; resident mode) keep every token's x in
// shared memory, and with RouteIn the kernel also routes them itself: each
// CTA sums the router's partial logits, selects (route_select.cuh) and
// groups in shared memory.  The combine is fused in: each CTA owns a range
// of output columns (about n / CTAs) and streams those rows of every active
// expert, concatenated, in full 8-row slabs (a slab may span two experts:
// the mma computes every row against every token anyway).  A reducer warp
// sums the consumers' partial tiles in warp order and keeps the slab's
// SiLU(8 x 8) tile in shared memory as it is; at the end it sums the slots
// of every token for its columns, so nothing leaves the CTA but v.
// Otherwise (fp32, or more tokens) the rows of all active experts, in whole
// slabs of one expert, are split evenly over the CTAs, the consumers reduce
// each slab's partial tiles themselves and its results go to P.
// Every wait is bounded; a wait that runs out sets MOVA_ERR_TIMEOUT in the
// status block and the CTA drains its copies and exits.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "internal.h"
#include "route_select.cuh"

#include "sm100.cuh"

namespace mova {

// The one-launch decode kernel's grid-barrier words: library-owned device
// memory, zero when the module loads.  Each launch takes the next slot of
// the ring, so consecutive launches on a stream use different words, and a
// completed barrier leaves its word as it found it (the top bit flipped).
constexpr int kGridBarSlots = 64;
__device__ unsigned int g_grid_bar[kGridBarSlots];

namespace {

constexpr int kConsumerWarps = 8;
// Warp 8 produces; warp 9 reduces the consumers' partial tiles in resident
// (decode) mode.
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kReducerWarp = kConsumerWarps + 1;
constexpr int kThreads = (kConsumerWarps + 2) * 32;
constexpr int kRowsPerStage = kConsumerWarps;
constexpr int kTok = 8;
constexpr int kMaxStages = 8;
// More stages than this do not raise the streaming rate: the extra requests
// in flight only queue in the memory system.
constexpr int kStreamStages = 4;

// Resident mode (bf16, T <= 8): the x rows of all tokens stay in shared
// memory for the whole kernel.
__host__ __device__ constexpr bool is_resident(bool mma, int T) { return mma && T <= kTok; }

template <typename DT> struct Vec;
template <> struct Vec<__nv_bfloat16> { static constexpr int EL = 8; };
template <> struct Vec<float> { static constexpr int EL = 4; };

__device__ __forceinline__ void unpack(const uint4& u, const __nv_bfloat16*, float out[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void unpack(const uint4& u, const float*, float out[4]) {
  out[0] = __uint_as_float(u.x); out[1] = __uint_as_float(u.y);
  out[2] = __uint_as_float(u.z); out[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void load_x(const __nv_bfloat16* p, float out[8]) { load8(p, out); }
__device__ __forceinline__ void load_x(const float* p, float out[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
}

// ---- bf16 consumers: legacy mma.sync m16n8k16 fragments ------------------
// A = 8 weight rows (rows 8..15 of the fragment are zero), B = up to 8
// tokens' x, both read with ldmatrix from row-padded shared memory (pitch =
// row bytes + 16, so the 8 rows of an 8x8 matrix hit distinct banks).  The 8
// consumer warps split K; partial 8x8 tiles meet in shared memory and are
// summed in warp order.

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

// Consumer-group barrier (the 8 consumer warps only; the producer warp never
// joins it).
// Partial-tile buffers of the consumer warps: one per stage slot (resident
// mode), at least the two that alternate otherwise.
__host__ __device__ constexpr int red_slots(int NS) { return NS > 2 ? NS : 2; }

__device__ __forceinline__ void consumers_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Grid-wide barrier of a launch whose CTAs are all resident (one per SM):
// CTA 0 adds 2^31 - (G - 1) to the word and every other CTA adds 1, so the
// word's top bit flips exactly when the last CTA arrives, whatever the order
// and whatever the top bit was, and the low bits return to where they were.
// Thread 0 of each CTA waits (bounded) for the flip; false if the wait ran
// out.  skip_arrive (a test-only fault) keeps this CTA from arriving.
__device__ __forceinline__ bool grid_barrier(unsigned int* word, long long limit, bool skip_arrive,
                                             volatile int* ok_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    const unsigned int add = blockIdx.x == 0 ? 0x80000000u - (gridDim.x - 1) : 1u;
    const unsigned int old = skip_arrive ? *reinterpret_cast<volatile unsigned int*>(word) : atomicAdd(word, add);
    const long long start = clock64();
    while (((*reinterpret_cast<volatile unsigned int*>(word) ^ old) & 0x80000000u) == 0) {
      if (clock64() - start > limit) {
        ok = 0;
        break;
      }
    }
    __threadfence();
    *ok_smem = ok;
  }
  __syncthreads();
  return *ok_smem != 0;
}

template <typename DT>
__global__ void __launch_bounds__(kThreads, 1)
stream_experts_kernel(const DT* __restrict__ x, const DT* __restrict__ Wv,
                      const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets,
                      const int32_t* __restrict__ perm, const float* __restrict__ w32,
                      const int32_t* __restrict__ active, StatusBlock* __restrict__ sb, int T,
                      int d, int n, int k, float* __restrict__ P, int NS,
                      DT* __restrict__ v, RouteIn route,
                      StreamFault fault, long long ldw, bool resident) {
  constexpr bool kMma = sizeof(DT) == 2;
  constexpr int EL = Vec<DT>::EL;
  extern __shared__ __align__(128) uint8_t smem[];
  const size_t row_bytes = static_cast<size_t>(d) * sizeof(DT);
  const size_t pitch = row_bytes + 16;
  const size_t stage_bytes = pitch * kRowsPerStage;
  uint8_t* stages = smem;
  uint8_t* xs = smem + NS * stage_bytes;  // bf16: kTok padded x rows
  // Partial tiles of the consumer warps: one [warps][8][8] buffer per stage
  // slot in resident mode, two alternating ones otherwise.
  float* red = reinterpret_cast<float*>(xs + (kMma ? kTok * pitch : 0));
  float* tok_w = red + (kMma ? red_slots(NS) * kConsumerWarps * 64 : 0);  // weights of the staged pairs
  int* tok_p = reinterpret_cast<int*>(tok_w + kTok);           // their grouped positions
  // Resident mode: every token's x row stays in the x tile for the whole
  // kernel (the mma computes all 8 token columns for every expert; the final
  // combine reads each pair's token column), and the tables below replace
  // all global loads of the grouping.
  int* slot_act = tok_p + kTok;                             // [64] active-list index of pair f's expert
  int* act_cnt = slot_act + 64;                             // [64] pairs per active expert
  int* act_off = act_cnt + 64;                              // [64] first position
  float* slot_w = reinterpret_cast<float*>(act_off + 64);  // [64] weight of pair f
  uint64_t* full = reinterpret_cast<uint64_t*>(slot_w + 64);
  uint64_t* empty = full + kMaxStages;
  uint64_t* xbar = empty + kMaxStages;  // resident x rows landed
  uint64_t* partb = xbar + 2;           // [kMaxStages] resident: a stage's 8 partial tiles are in red
  int* act = reinterpret_cast<int*>(partb + kMaxStages);
  volatile int* abort_flag = act + 64;
  int* issued = act + 65;
  // Resident mode: the SiLU values of this CTA's rows, [flat row][token].
  float* hv = reinterpret_cast<float*>(act + 68);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Resident mode: this CTA's output columns [r_lo, r_lo + nr), formed here,
  // off the path from the selection to the first weight copy (n * CTAs
  // stays far below 2^32).
  const int r_lo = static_cast<int>(static_cast<unsigned>(n) * blockIdx.x / gridDim.x);
  const int nr = static_cast<int>(static_cast<unsigned>(n) * (blockIdx.x + 1) / gridDim.x) - r_lo;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      // Resident mode: the reducer frees a stage; otherwise the consumers.
      mbar_init(&empty[s], resident ? 1 : kConsumerWarps);
      mbar_init(&partb[s], kConsumerWarps);
    }
    *abort_flag = 0;
    *issued = 0;
    fence_barrier_init();
  }
  // One-launch decode: CTAs below E * S each compute one (expert, K range)
  // of the partial logits; the first chunk of the router row is requested
  // before the grid dependency wait (no kernel writes router weights).
  const bool one_launch = route.Wr != nullptr;
  const int lg_units = one_launch ? route.E * route.S : 0;
  const bool lg_cta = static_cast<int>(blockIdx.x) < lg_units && threadIdx.x < kPartThreads;
  int lg_e = 0, lg_c0 = 0, lg_ce = 0;
  float lg_w0[8];
  if (lg_cta) {
    lg_e = blockIdx.x % route.E;
    const int rs = blockIdx.x / route.E;
    const int chunks = d / 8;
    lg_ce = chunks * (rs + 1) / route.S;
    lg_c0 = chunks * rs / route.S + threadIdx.x;
    if (lg_c0 < lg_ce) load8(route.Wr + static_cast<size_t>(lg_e) * d + 8 * lg_c0, lg_w0);
  }
  pdl_wait();  // the previous kernel on the stream is complete (two-launch: routing of this call)
  if (resident && threadIdx.x == kReducerWarp * 32) {
    // The resident x tile: one bulk copy per token row, issued at once so its
    // latency overlaps the first weight stages.  The reducer warp, idle until
    // the first stage, initialises its barrier and issues the copies, so the
    // selecting warps do not wait for the issue; the consumers wait on the
    // barrier only after the grouping barrier, which this warp joins later.
    mbar_init(xbar, 1);
    fence_barrier_init();
    const uint32_t row_bytes_x = static_cast<uint32_t>(row_bytes);
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(T) * row_bytes_x);
    for (int t = 0; t < T; ++t)
      bulk_g2s(xs + t * pitch, x + static_cast<size_t>(t) * d, row_bytes_x, xbar, policy_evict_last());
  }
  if (one_launch) {
    // The partial logits of this call (the part of the logits kernel of the
    // two-launch path), then the status reset, then one grid
    // barrier: after it every CTA reads all of them.
    __shared__ int gb_ok;
    float* lred = red;  // free until the weight stream starts
    for (int unit = blockIdx.x; unit < lg_units; unit += gridDim.x) {
      if (threadIdx.x < kPartThreads) {
        const float* wrow = route.Wr + static_cast<size_t>(unit % route.E) * d;
        const int rs = unit / route.E;
        const int chunks = d / 8;
        const int ce = chunks * (rs + 1) / route.S;
        const int c0 = chunks * rs / route.S + threadIdx.x;
        float w0[8];
        if (unit == static_cast<int>(blockIdx.x) && lg_cta) {
#pragma unroll
          for (int q = 0; q < 8; ++q) w0[q] = lg_w0[q];
        } else if (c0 < ce) {
          load8(wrow + 8 * c0, w0);
        }
        partial_logits_warp(wrow, x, T, d, c0, ce, w0, lane, warp, lred);
        consumers_sync();
        if (threadIdx.x < kTok)
          route.part_out[(rs * kTok + threadIdx.x) * 64 + unit % route.E] = partial_logits_final(lred, threadIdx.x);
        consumers_sync();
      }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      sb->code = 0;
      sb->detail = 0;
      sb->work_next = 0;
    }
    if (!grid_barrier(&g_grid_bar[route.bar_slot], fault.wait_limit, fault.skip_barrier && blockIdx.x == 0,
                      &gb_ok)) {
      if (threadIdx.x == 0) {
        raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
      }
    }
    __syncthreads();
  }
  // Route mode: the consumer warps select and group the batch from the
  // partial logits (every CTA the same, in the same fixed order).
  __shared__ int r_sel[kTok * 8];
  __shared__ float r_w[kTok * 8];
  __shared__ int r_scratch[128];
  __shared__ int32_t r_cnt[64], r_off[65], r_pos[64], r_perm[64];
  __shared__ int r_nact;
  __shared__ int p_act[64];  // the producer's own copy of the active list (route mode)
  int p_nact = 0;
  const bool routing = route.part != nullptr;
  if (routing) {
    if (threadIdx.x < kConsumerWarps * 32) {
      // Warp t selects token t straight from the partials: lane l loads
      // experts l and l + 32 of every K range (all loads issued before the
      // first is used: one L2 round trip) and sums them in range order.
      static_assert(kTok <= kConsumerWarps, "a warp per token");
      if (warp < T) {
        float p0[kMaxLogitSplits], p1[kMaxLogitSplits];
#pragma unroll
        for (int r = 0; r < kMaxLogitSplits; ++r) {
          const float* pr = route.part + (r * kTok + warp) * 64;
          p0[r] = r < route.S ? __ldcg(pr + lane) : 0.f;
          p1[r] = r < route.S ? __ldcg(pr + lane + 32) : 0.f;
        }
        const float b0 = lane < route.E ? route.br[lane] : 0.f;
        const float b1 = lane + 32 < route.E ? route.br[lane + 32] : 0.f;
        float l0 = p0[0], l1 = p1[0];
#pragma unroll
        for (int r = 1; r < kMaxLogitSplits; ++r) {
          if (r < route.S) {
            l0 += p0[r];
            l1 += p1[r];
          }
        }
        int es[8];
        float ss[8];
        select_top_k_regs(l0, l1, b0, b1, route.E, k, lane, es, ss);
        store_selection(es, ss, k, route.scale, warp, lane, r_sel, r_w,
                        blockIdx.x == 0 ? route.idx_out : nullptr, route.w_out);
      }
      consumers_sync();
      // The selection is complete: the producer warp may derive the active
      // experts and start the weight stream while warp 0 groups the pairs.
      asm volatile("bar.arrive 3, %0;" ::"n"((kConsumerWarps + 1) * 32) : "memory");
      if (warp == 0) {
        const int na = group_pairs_warp(r_sel, T * k, route.E, lane, r_scratch, r_cnt, r_off, r_pos,
                                        r_perm, act);
        if (lane == 0) r_nact = na;
        if (blockIdx.x == 0 && route.counts_out != nullptr) {
          // Every CTA groups the batch identically; CTA 0 also leaves the
          // result in global memory (counts, offsets, perm, pos, active).
          __syncwarp();
          for (int i = lane; i < route.E; i += 32) {
            route.counts_out[i] = r_cnt[i];
            route.offsets_out[i] = r_off[i];
          }
          if (lane == 0) {
            route.offsets_out[route.E] = r_off[route.E];
            sb->num_active = na;
          }
          for (int i = lane; i < T * k; i += 32) {
            route.perm_out[i] = r_perm[i];
            route.pos_out[i] = r_pos[i];
          }
          for (int i = lane; i < na; i += 32) route.active_out[i] = act[i];
        }
      }
    }
    if (warp == kProducerWarp) {
      // The active experts (ascending), from the selection alone: the same
      // list the grouping builds.
      asm volatile("bar.sync 3, %0;" ::"n"((kConsumerWarps + 1) * 32) : "memory");
      // Experts 0-31 and 32-63 as two 32-bit masks, each OR-reduced over
      // the warp in one instruction.
      uint32_t m_lo = 0, m_hi = 0;
      for (int i = lane; i < T * k; i += 32) {
        const int e = r_sel[i];
        if (e < 32) m_lo |= 1u << e; else m_hi |= 1u << (e - 32);
      }
      m_lo = __reduce_or_sync(0xffffffffu, m_lo);
      m_hi = __reduce_or_sync(0xffffffffu, m_hi);
      const uint64_t m = (static_cast<uint64_t>(m_hi) << 32) | m_lo;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = lane + 32 * h;
        if ((m >> e) & 1ull) p_act[__popcll(m & ((1ull << e) - 1ull))] = e;
      }
      p_nact = __popcll(m);
      __syncwarp();
    }
  } else {
    const int na = sb->num_active;
    if (threadIdx.x < 64) act[threadIdx.x] = (threadIdx.x < na) ? active[threadIdx.x] : 0;
  }
  // Route mode: the producer goes ahead; the other warps wait for the grouping.
  if (!routing)
    __syncthreads();
  else if (warp != kProducerWarp)
    asm volatile("bar.sync 4, %0;" ::"n"((kConsumerWarps + 1) * 32) : "memory");
  const int nact = routing ? (warp == kProducerWarp ? p_nact : r_nact) : sb->num_active;
  const int* act_p = routing && warp == kProducerWarp ? p_act : act;
  pdl_trigger();

  // Resident mode (the combine fused in): this CTA owns output columns
  // [r_lo, r_lo + nr).  Its rows are those columns of every active expert in
  // turn -- flat row f is column r_lo + f % nr of active expert f / nr --
  // and stage j holds flat rows 8j .. 8j + 7.
  // Otherwise the rows of all active experts, in units of whole stages
  // (n % 8 == 0, so a stage never straddles two experts), are split evenly
  // over the CTAs, expert-major, so the staged x rows change only with the
  // expert.
  const int units_per_expert = n / kRowsPerStage;
  const int rows_total = nact * nr;
  const int units = resident ? (rows_total + kRowsPerStage - 1) / kRowsPerStage : nact * units_per_expert;
  const int u0 = resident ? 0 : static_cast<int>(static_cast<long long>(units) * blockIdx.x / gridDim.x);
  const int u1 = resident ? units : static_cast<int>(static_cast<long long>(units) * (blockIdx.x + 1) / gridDim.x);
  const int nstages = u1 - u0;

  if (warp == kProducerWarp) {
    // The producer warp runs the loop together; lane 0 declares each stage's
    // bytes, then lanes 0-7 issue one row copy each, so a stage's eight
    // copies leave at once.  The unit's expert and row advance incrementally.
    const uint64_t pol = policy_evict_first();
    int s = 0;
    uint32_t phase = 0;
    int j = 0;
    for (; j < nstages; ++j) {
      if (j >= NS &&
          !__all_sync(0xffffffffu, mbar_wait_or_abort(&empty[s], phase ^ 1, abort_flag, fault.wait_limit))) {
        if (lane == 0 && *abort_flag == 0) {
          raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
          *abort_flag = 1;
        }
        break;
      }
      if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
      // Test-only injection: CTA 0 stops issuing here, so the consumers'
      // wait for this stage must run out.
      if (j == fault.stall_stage && blockIdx.x == 0) break;
      // This lane's row of the stage: active expert a, row r.
      int nrows = kRowsPerStage, a, r;
      if (resident) {
        const int f = j * kRowsPerStage + lane;
        nrows = min(kRowsPerStage, rows_total - j * kRowsPerStage);
        a = f / max(nr, 1);
        r = r_lo + (f - a * nr);
      } else {
        const int u = u0 + j;
        a = u / units_per_expert;
        r = (u - a * units_per_expert) * kRowsPerStage + lane;
      }
      uint8_t* dst = stages + s * stage_bytes;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nrows * row_bytes));
      __syncwarp();
      if (lane < nrows)
        bulk_g2s(dst + lane * pitch, Wv + (static_cast<size_t>(act_p[a]) * ldw + r) * d,
                 static_cast<uint32_t>(row_bytes), &full[s], pol);
      __syncwarp();
      if (++s == NS) { s = 0; phase ^= 1; }
    }
    if (lane == 0) *issued = j;
  } else if (warp == kReducerWarp) {
    if (resident) {
      // Resident mode: the consumer warps hand each stage's partial tiles
      // (their K slices of 8 weight rows x 8 token columns) over through an
      // mbarrier instead of meeting at a block barrier; this warp sums them
      // in warp order, applies SiLU, keeps the stage's rows of every pair of
      // its expert, and frees the stage.  It takes every stage, even after a
      // failure (then keeping nothing), so the stage ring stays in step.
      bool all_ok = true;
      for (int j = 0; j < nstages; ++j) {
        const int s = j % NS;
        bool ok = *abort_flag == 0;
        if (ok && !mbar_wait_or_abort(&partb[s], (j / NS) & 1, abort_flag, fault.wait_limit)) {
          ok = false;
          if (*abort_flag == 0) {
            raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
            *abort_flag = 1;
          }
        }
        ok = __all_sync(0xffffffffu, ok);
        all_ok = all_ok && ok;
        if (ok) {
          // Stage row q (flat row 8j + q), token column c: hv[(8j + q) * 8 + c].
          const float* rb = red + s * (kConsumerWarps * 64);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int e = lane + 32 * h;  // row e / 8, token column e % 8
            float acc = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) acc += rb[w * 64 + e];
            hv[j * 64 + e] = siluf_(acc);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      // Every stage of every active expert is in (a role that failed set the
      // abort flag before its last arrival, so it is seen here): the combine
      // for this CTA's columns,
      //   v[t, r] = sum over slots (ascending) of w[t, slot] * SiLU value,
      // the same fmaf chain as the separate combine pass.
      if (all_ok && *abort_flag == 0) {
        for (int i = lane; i < T * nr; i += 32) {
          const int t = i / nr;
          const int r = i - t * nr;
          float acc = 0.f;
          for (int sl = 0; sl < k; ++sl) {
            const int f = t * k + sl;
            acc = fmaf(slot_w[f], hv[(slot_act[f] * nr + r) * 8 + t], acc);
          }
          v[static_cast<size_t>(t) * n + r_lo + r] = from_f32<DT>(acc);
        }
      }
    }
  } else {
    int cur_a = -1, cnt = 0, off = 0;
    int staged_a = -1, staged_c0 = -1;  // whose x rows the x tile holds
    int rbuf = 0;
    const int ksteps = d / 16;
    const int kb = ksteps * warp / kConsumerWarps;
    const int ke = ksteps * (warp + 1) / kConsumerWarps;
    if (resident) {
      // Pair tables, while x and the first weight stages are in flight.
      const int N = T * k;
      if (threadIdx.x < N) slot_w[threadIdx.x] = routing ? r_w[threadIdx.x] : w32[threadIdx.x];
      if (threadIdx.x < nact) {
        const int e = act[threadIdx.x];
        const int cnt_e = routing ? r_cnt[e] : counts[e];
        const int off_e = routing ? r_off[e] : offsets[e];
        act_cnt[threadIdx.x] = cnt_e;
        act_off[threadIdx.x] = off_e;
        for (int i = 0; i < cnt_e; ++i) slot_act[routing ? r_perm[off_e + i] : perm[off_e + i]] = threadIdx.x;
      }
      if (!mbar_wait_or_abort(xbar, 0, abort_flag, fault.wait_limit)) {
        raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
        *abort_flag = 1;
      }
      consumers_sync();
    }
    // Every consumer warp runs every stage of the loop and meets the others
    // at the same barriers, whatever happens: after a failed wait (or an
    // abort raised by another role) a warp skips the stage's arithmetic but
    // not its barriers, so no warp can be left waiting at one.  `ok` is
    // warp-uniform (the mma.sync path needs the whole warp).
    for (int j = 0; j < nstages; ++j) {
      const int s = j % NS;
      bool ok = *abort_flag == 0;
      if (ok && !mbar_wait_or_abort(&full[s], (j / NS) & 1, abort_flag, fault.wait_limit)) {
        ok = false;
        if (*abort_flag == 0) {
          raise_status(sb, MOVA_ERR_TIMEOUT, blockIdx.x);
          *abort_flag = 1;
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      const uint8_t* wst = stages + s * stage_bytes;
      if constexpr (kMma) {
        if (resident) {
          // The stage's (8 weight rows) x (8 token columns) tile over this
          // warp's K slice, with four independent accumulators fed by four
          // k-steps of loads at a time (summed in a fixed order at the end),
          // handed to the reducer warp.
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          if (ok) {
            const int lr = lane & 7;
            const int lk = (lane >> 3) & 1;
            const uint32_t a_base = smem_u32(wst) + lr * static_cast<uint32_t>(pitch) + lk * 16;
            const uint32_t b_base = smem_u32(xs) + lr * static_cast<uint32_t>(pitch) + lk * 16;
            float c1[4] = {0.f, 0.f, 0.f, 0.f}, c2[4] = {0.f, 0.f, 0.f, 0.f}, c3[4] = {0.f, 0.f, 0.f, 0.f};
            int ks = kb;
            for (; ks + 3 < ke; ks += 4) {
              uint32_t a0[4], a2[4], b0[4], b1[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                ldsm_x2(a_base + (ks + q) * 32, a0[q], a2[q]);
                ldsm_x2(b_base + (ks + q) * 32, b0[q], b1[q]);
              }
              mma_bf16_16816(acc, a0[0], a2[0], b0[0], b1[0]);
              mma_bf16_16816(c1, a0[1], a2[1], b0[1], b1[1]);
              mma_bf16_16816(c2, a0[2], a2[2], b0[2], b1[2]);
              mma_bf16_16816(c3, a0[3], a2[3], b0[3], b1[3]);
            }
            for (; ks < ke; ++ks) {
              uint32_t a0, a2, b0, b1;
              ldsm_x2(a_base + ks * 32, a0, a2);
              ldsm_x2(b_base + ks * 32, b0, b1);
              mma_bf16_16816(acc, a0, a2, b0, b1);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = (acc[q] + c1[q]) + (c2[q] + c3[q]);
          }
          // acc[0], acc[1]: weight row lane / 4, token columns 2 * (lane % 4) + {0, 1}.
          float* rb = red + s * (kConsumerWarps * 64);
          const int g = lane >> 2;
          const int tc = (lane & 3) * 2;
          rb[warp * 64 + g * 8 + tc] = acc[0];
          rb[warp * 64 + g * 8 + tc + 1] = acc[1];
          __syncwarp();
          if (lane == 0) mbar_arrive(&partb[s]);
          continue;  // the reducer frees the stage
        }
      }
      const int a = (u0 + j) / units_per_expert;
      const int r0 = (u0 + j - a * units_per_expert) * kRowsPerStage;
      if (a != cur_a) {
        cur_a = a;
        cnt = counts[act[a]];
        off = offsets[act[a]];
      }
      for (int c0 = 0; c0 < cnt; c0 += kTok) {
        const int nt = min(kTok, cnt - c0);
        if constexpr (kMma) {
          // Stage this chunk's x rows (once per expert and chunk; rows
          // beyond nt repeat the last token and are never stored).
          if (!resident && (a != staged_a || c0 != staged_c0)) {
            staged_a = a;
            staged_c0 = c0;
            consumers_sync();
            const int vec_per_row = static_cast<int>(row_bytes / 16);
            for (int i = threadIdx.x; i < kTok * vec_per_row; i += kConsumerWarps * 32) {
              const int t = i / vec_per_row;
              const int v = i - t * vec_per_row;
              const int f = perm[off + c0 + min(t, nt - 1)];
              const uint4* srow = reinterpret_cast<const uint4*>(x + static_cast<size_t>(f / k) * d);
              *reinterpret_cast<uint4*>(xs + t * pitch + v * 16) = srow[v];
            }
            if (threadIdx.x < kTok) {
              const int t = threadIdx.x;
              const int p = off + c0 + min(t, nt - 1);
              tok_p[t] = p;
              tok_w[t] = w32[perm[p]];
            }
            consumers_sync();
          }
          // This warp's K slice, in 16-element steps.
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
          const int lr = lane & 7;
          const int lk = (lane >> 3) & 1;
          const uint32_t a_base = smem_u32(wst) + lr * static_cast<uint32_t>(pitch) + lk * 16;
          const uint32_t b_base = smem_u32(xs) + lr * static_cast<uint32_t>(pitch) + lk * 16;
          if (ok) {
#pragma unroll 4
            for (int ks = kb; ks < ke; ++ks) {
              uint32_t a0, a2, b0, b1;
              ldsm_x2(a_base + ks * 32, a0, a2);
              ldsm_x2(b_base + ks * 32, b0, b1);
              mma_bf16_16816(acc, a0, a2, b0, b1);
            }
          }
          // acc[0], acc[1]: weight row lane/4, tokens 2*(lane%4) + {0, 1}.
          // Two reduction buffers alternate, so one barrier per tile
          // suffices: a warp can only overwrite a buffer after every thread
          // has passed the next barrier, i.e. finished reading it.
          float* rb = red + (rbuf & 1) * (kConsumerWarps * 64);
          ++rbuf;
          const int g = lane >> 2;
          const int tc = (lane & 3) * 2;
          rb[(warp * 8 + g) * 8 + tc] = acc[0];
          rb[(warp * 8 + g) * 8 + tc + 1] = acc[1];
          consumers_sync();
          if (threadIdx.x < 64) {
            const int row = threadIdx.x >> 3;
            const int t = threadIdx.x & 7;
            if (t < nt) {
              const int col = t;  // the pair's token column
              float h = 0.f;
#pragma unroll
              for (int w = 0; w < kConsumerWarps; ++w) h += rb[(w * 8 + row) * 8 + col];
              const int p = resident ? off + c0 + t : tok_p[t];
              P[static_cast<size_t>(p) * n + r0 + row] = siluf_(h);
            }
          }
        } else if (ok) {
          // fp32 weights: CUDA-core dot products, one row per warp.
          const int f_last = nt - 1;
          const DT* xr[kTok];
#pragma unroll
          for (int t = 0; t < kTok; ++t) {
            const int f = perm[off + c0 + min(t, f_last)];
            xr[t] = x + static_cast<size_t>(f / k) * d;
          }
          const uint8_t* wrow = wst + warp * pitch;
          float acc[kTok];
#pragma unroll
          for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
          for (int kk = lane * EL; kk < d; kk += 32 * EL) {
            const uint4 uu = *reinterpret_cast<const uint4*>(wrow + kk * sizeof(DT));
            float wv[EL];
            unpack(uu, static_cast<const DT*>(nullptr), wv);
#pragma unroll
            for (int t = 0; t < kTok; ++t) {
              if (t < nt) {
                float xv[EL];
                load_x(xr[t] + kk, xv);
#pragma unroll
                for (int q = 0; q < EL; ++q) acc[t] = fmaf(wv[q], xv[q], acc[t]);
              }
            }
          }
          float mine = 0.f;
#pragma unroll
          for (int t = 0; t < kTok; ++t) {
            if (t < nt) {
#pragma unroll
              for (int o = 16; o >= 1; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
              if (lane == t) mine = acc[t];
            }
          }
          if (lane < nt) {
            const int p = off + c0 + lane;
            P[static_cast<size_t>(p) * n + r0 + warp] = siluf_(mine);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
  __syncthreads();
  // No bulk copy may still be writing this CTA's shared memory at exit: wait
  // (bounded) for the last phase issued into every stage.
  if (threadIdx.x == kProducerWarp * 32) {
    const int done = *issued;
    for (int j = max(0, done - NS); j < done; ++j) mbar_wait(&full[j % NS], (j / NS) & 1);
    if (resident) mbar_wait(xbar, 0);
  }
}

}  // namespace

namespace {
std::atomic<unsigned int> g_bar_next{0};
}  // namespace

int next_grid_barrier_slot() { return static_cast<int>(g_bar_next.fetch_add(1) % kGridBarSlots); }

cudaError_t reset_grid_barriers(cudaStream_t stream) {
  void* p = nullptr;
  cudaError_t err = cudaGetSymbolAddress(&p, g_grid_bar);
  if (err != cudaSuccess) return err;
  return cudaMemsetAsync(p, 0, sizeof(g_grid_bar), stream);
}

namespace {

// Resident mode's buffer of SiLU values: a CTA's rows (its ceil(n / CTAs)
// columns of each of at most min(E, T k) active experts, in whole stages)
// for all 8 token columns.
size_t hv_bytes_for(int T, int n, int k, int E) {
  const int G = sm_count();
  const size_t rows = static_cast<size_t>(std::min(E, T * k)) * ((n + G - 1) / G);
  return (rows + kRowsPerStage - 1) / kRowsPerStage * kRowsPerStage * kTok * sizeof(float);
}

// Shared memory of a launch in the given mode: the most stages (up to
// kStreamStages) that fit next to the fixed parts, whose partial-tile buffers
// grow with the stage count; 0 if not even two fit.
size_t smem_bytes(int d, bool mma, size_t hv_bytes, int* stages_out) {
  const size_t pitch = static_cast<size_t>(d) * (mma ? 2 : 4) + 16;
  const size_t stage_bytes = pitch * kRowsPerStage;
  // With the kernel's ~2.4 KB of static arrays, under the 227 KB a block
  // may opt in to.
  const size_t budget = 222 * 1024;
  for (int NS = kStreamStages; NS >= 2; --NS) {
    const size_t fixed = (mma ? kTok * pitch + red_slots(NS) * kConsumerWarps * 64 * sizeof(float) : 0) +
                         2 * kTok * sizeof(float) + 4 * 64 * sizeof(int) +
                         (3 * kMaxStages + 2) * sizeof(uint64_t) + 68 * sizeof(int) + hv_bytes;
    if (NS * stage_bytes + fixed <= budget) {
      if (stages_out) *stages_out = NS;
      return NS * stage_bytes + fixed;
    }
  }
  if (stages_out) *stages_out = 0;
  return 0;
}

}  // namespace

bool stream_resident(int T, int d, int n, int k, int E, mova_dtype dt) {
  const bool mma = dt == MOVA_BF16;
  return is_resident(mma, T) && smem_bytes(d, mma, hv_bytes_for(T, n, k, E), nullptr) != 0;
}

size_t stream_experts_smem(int d, mova_dtype dt, int T, int n, int k, int E, int* stages_out) {
  const bool res = stream_resident(T, d, n, k, E, dt);
  return smem_bytes(d, dt == MOVA_BF16, res ? hv_bytes_for(T, n, k, E) : 0, stages_out);
}

cudaError_t launch_stream_experts(const void* x, const void* Wv, long long ldw, mova_dtype dt,
                                  const int32_t* counts,
                                  const int32_t* offsets, const int32_t* perm, const float* w32,
                                  const int32_t* active, StatusBlock* sb, int T, int d, int n,
                                  int k, int E, float* P, void* v, const RouteIn& route,
                                  cudaStream_t stream) {
  int NS = 0;
  const size_t smem = stream_experts_smem(d, dt, T, n, k, E, &NS);
  if (smem == 0) return cudaErrorInvalidValue;
  // Resident mode always combines inside the kernel, and only it routes.
  const bool resident = stream_resident(T, d, n, k, E, dt);
  if (resident != (v != nullptr) || (!resident && route.part != nullptr)) return cudaErrorInvalidValue;
  const dim3 grid(sm_count());
  const StreamFault fault = take_stream_fault();
  if (dt == MOVA_BF16) {
    auto kern = stream_experts_kernel<__nv_bfloat16>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(kern, grid, dim3(kThreads), smem, stream,
                      static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(Wv),
                      counts, offsets, perm, w32, active, sb, T, d, n, k, P, NS,
                      static_cast<__nv_bfloat16*>(v), route, fault, ldw, resident);
  }
  auto kern = stream_experts_kernel<float>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(kern, grid, dim3(kThreads), smem, stream, static_cast<const float*>(x),
                    static_cast<const float*>(Wv), counts, offsets, perm, w32, active, sb, T, d, n,
                    k, P, NS, static_cast<float*>(v), route, fault, ldw, resident);
}

}  // namespace mova
