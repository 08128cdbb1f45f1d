// Gate, top-k selection and grouping of a few tokens by warps, shared by the
// router kernels and the weight-streaming kernel (which routes decode batches
// itself).  "MoVA: routing the value vectors, and why the KV cache does not
// notice", section "Where the routing happens": sigmoid gate on the router
// logits, the bias handed separately steers the top-k choice only, the k
// selected sigmoid scores are renormalised and multiplied by the scale.
#pragma once

#include "common.cuh"

namespace mova {

// Order-preserving map of a float to an unsigned key: a < b (as floats, no
// NaN) iff key(a) < key(b).  Every key of a float is >= key(-inf) =
// 0x007FFFFF, so 0 can mark a candidate that is taken or does not exist.
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Gate and selection of one token by one warp.  lg: the token's E logits,
// brs: the E biases (both in shared memory).  Lane l holds experts l and
// l + 32.  Each of the k rounds takes the warp maximum of the biased scores
// s + br (one redux.sync on order-preserving keys; a NaN score counts as
// -inf and never displaces a finite one), then the lowest expert index that
// attains it (ties go to the lower index), and retires that expert.  On
// return every lane holds the same sel_e / sel_s (unbiased sigmoid scores)
// for j < k.
// The same from the lane's two logits and biases in registers (experts
// lane and lane + 32; values of experts >= E are ignored).
__device__ __forceinline__ void select_top_k_regs(float lg0, float lg1, float br0, float br1, int E,
                                                  int k, int lane, int (&sel_e)[8], float (&sel_s)[8]) {
  const int e0 = lane, e1 = lane + 32;
  float s0 = 0.f, s1 = 0.f;
  uint32_t key0 = 0, key1 = 0;
  if (e0 < E) {
    s0 = sigmoidf_(lg0);
    const float b = s0 + br0;
    key0 = order_key(b == b ? b : -INFINITY);
  }
  if (e1 < E) {
    s1 = sigmoidf_(lg1);
    const float b = s1 + br1;
    key1 = order_key(b == b ? b : -INFINITY);
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k) {
      const uint32_t m = __reduce_max_sync(0xffffffffu, max(key0, key1));
      const unsigned c0 = __ballot_sync(0xffffffffu, key0 == m);
      const unsigned c1 = __ballot_sync(0xffffffffu, key1 == m);
      const int be = c0 ? __ffs(c0) - 1 : 32 + __ffs(c1) - 1;  // k <= E: always a live expert
      sel_e[j] = be;
      sel_s[j] = __shfl_sync(0xffffffffu, be < 32 ? s0 : s1, be & 31);
      if (be == e0) key0 = 0;
      if (be == e1) key1 = 0;
    }
  }
}

__device__ __forceinline__ void select_top_k(const float* lg, const float* brs, int E, int k,
                                             int lane, int (&sel_e)[8], float (&sel_s)[8]) {
  const int e0 = lane, e1 = lane + 32;
  select_top_k_regs(e0 < E ? lg[e0] : 0.f, e1 < E ? lg[e1] : 0.f, e0 < E ? brs[e0] : 0.f,
                    e1 < E ? brs[e1] : 0.f, E, k, lane, sel_e, sel_s);
}

// Sum of the k selected scores in slot order.
__device__ __forceinline__ float sum_k(const float (&s)[8], int k) {
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k) acc += s[j];
  return acc;
}

// Selection of token t by one warp from the selected experts and scores:
// written to shared memory, sel[t*k + j] (expert) and wsel[t*k + j]
// (renormalised, scaled weight); with idx_out / w_out non-null also to
// global memory.
__device__ __forceinline__ void store_selection(const int (&es)[8], const float (&ss)[8], int k, float scale,
                                                int t, int lane, int* sel, float* wsel, int32_t* idx_out,
                                                float* w_out) {
  const float ssum = sum_k(ss, k);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < k && lane == j) {
      const float wj = scale * ss[j] / ssum;
      sel[t * k + j] = es[j];
      wsel[t * k + j] = wj;
      if (idx_out != nullptr) {
        idx_out[t * k + j] = es[j];
        w_out[t * k + j] = wj;
      }
    }
  }
}

__device__ __forceinline__ void select_token(const float* lg, const float* brs, int E, int k,
                                             float scale, int t, int lane, int* sel, float* wsel,
                                             int32_t* idx_out, float* w_out) {
  int es[8];
  float ss[8];
  select_top_k(lg, brs, E, k, lane, es, ss);
  store_selection(es, ss, k, scale, t, lane, sel, wsel, idx_out, w_out);
}

// Partial router logits of decode batches (T <= 8): 256 threads (8 warps)
// sum one expert's router row against every token's x over a range of K.
// Thread i takes the 8-element chunks c0 = cb + i, c0 + 256, ... < ce (the
// first chunk's router weights w0 loaded by the caller, which may request
// them early), 8 fused multiply-adds per token in ascending element order.
// A transposing warp butterfly then leaves each token's warp sum in one lane
// group, written to red[warp * 8 + token]; after a barrier of the 256
// threads, partial_logits_final gives token t's sum (threads t < 8) with the
// warps' sums added in warp order.  Every step has a fixed order, so the
// partial logits do not depend on timing.
constexpr int kPartThreads = 256;
template <typename XT>
__device__ __forceinline__ void partial_logits_warp(const float* __restrict__ wrow, const XT* __restrict__ x,
                                                    int T, int d, int c0, int ce, const float (&w0)[8],
                                                    int lane, int warp, float* red) {
  float acc[8];
#pragma unroll
  for (int t = 0; t < 8; ++t) acc[t] = 0.f;
  for (int c = c0; c < ce; c += kPartThreads) {
    float w[8];
    if (c == c0) {
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = w0[q];
    } else {
      load8(wrow + 8 * c, w);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (t < T) {
        float xv[8];
        load8(x + static_cast<size_t>(t) * d + 8 * c, xv);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[t] = fmaf(w[q], xv[q], acc[t]);
      }
    }
  }
  // Transposing butterfly over the 8 token sums: after the steps with
  // offsets 16, 8, 4 lane l holds token 4*b4 + 2*b3 + b2 (bits of l) summed
  // over its 8-lane group pattern; offsets 2 and 1 finish the warp sum.
  const bool u16 = (lane & 16) != 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = u16 ? acc[i] : acc[i + 4];
    const float keep = u16 ? acc[i + 4] : acc[i];
    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  const bool u8 = (lane & 8) != 0;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = u8 ? acc[i] : acc[i + 2];
    const float keep = u8 ? acc[i + 2] : acc[i];
    acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const bool u4 = (lane & 4) != 0;
  const float send = u4 ? acc[0] : acc[1];
  const float keep = u4 ? acc[1] : acc[0];
  acc[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 2);
  acc[0] += __shfl_xor_sync(0xffffffffu, acc[0], 1);
  if ((lane & 3) == 0) red[warp * 8 + ((lane >> 4) & 1) * 4 + ((lane >> 3) & 1) * 2 + ((lane >> 2) & 1)] = acc[0];
}
__device__ __forceinline__ float partial_logits_final(const float* red, int t) {
  float v = red[t];
#pragma unroll
  for (int w = 1; w < kPartThreads / 32; ++w) v += red[w * 8 + t];
  return v;
}

// Grouping of N <= 64 pairs (pair f = token f / k, slot f % k, expert
// sel[f]) by expert, by one warp: a stable counting sort.  Lane l holds pairs
// l and l + 32; a pair's rank among the earlier pairs of its expert comes
// from the match mask of its half plus, for the second half, the first
// half's count of that expert.  Outputs (shared or global memory): cnt[e],
// off[e] (exclusive prefix, off[E] = N), pos[f] (grouped position of pair f),
// perm[p] (pair at grouped position p), act[i] (the experts with pairs, in
// ascending order).  scratch: 128 ints of shared memory.  Returns the number
// of active experts (on every lane).
__device__ __forceinline__ int group_pairs_warp(const int* sel, int N, int E, int lane, int* scratch,
                                                int32_t* cnt, int32_t* off, int32_t* pos,
                                                int32_t* perm, int32_t* act) {
  int* half0 = scratch;
  int* half1 = scratch + 64;
  half0[lane] = 0; half0[lane + 32] = 0;
  half1[lane] = 0; half1[lane + 32] = 0;
  __syncwarp();
  const int f0 = lane, f1 = lane + 32;
  const int ef0 = (f0 < N) ? sel[f0] : -1 - f0;
  const int ef1 = (f1 < N) ? sel[f1] : -1 - f1;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned m0 = __match_any_sync(0xffffffffu, ef0);
  const unsigned m1 = __match_any_sync(0xffffffffu, ef1);
  const int r0 = __popc(m0 & lt);
  const int r1 = __popc(m1 & lt);
  if (f0 < N && r0 == 0) half0[ef0] = __popc(m0);
  if (f1 < N && r1 == 0) half1[ef1] = __popc(m1);
  __syncwarp();
  const int cnt0 = half0[lane] + half1[lane];
  const int cnt1 = half0[lane + 32] + half1[lane + 32];
  const int rank0 = r0;
  const int rank1 = (f1 < N) ? half0[ef1] + r1 : 0;
  // Exclusive scan of the counts over experts lane, lane + 32.
  int inc0 = cnt0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc0, o);
    if (lane >= o) inc0 += y;
  }
  const int tot0 = __shfl_sync(0xffffffffu, inc0, 31);
  int inc1 = cnt1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, inc1, o);
    if (lane >= o) inc1 += y;
  }
  const int ex0 = inc0 - cnt0;
  const int ex1 = tot0 + inc1 - cnt1;
  __syncwarp();
  // The scratch now holds the offsets (read back below by other lanes).
  half0[lane] = ex0;
  half0[lane + 32] = ex1;
  if (lane < E) { cnt[lane] = cnt0; off[lane] = ex0; }
  if (lane + 32 < E) { cnt[lane + 32] = cnt1; off[lane + 32] = ex1; }
  if (lane == 0) off[E] = N;
  __syncwarp();
  if (f0 < N) { const int p = half0[ef0] + rank0; pos[f0] = p; perm[p] = f0; }
  if (f1 < N) { const int p = half0[ef1] + rank1; pos[f1] = p; perm[p] = f1; }
  const bool a0 = lane < E && cnt0 > 0;
  const bool a1 = lane + 32 < E && cnt1 > 0;
  const unsigned b0 = __ballot_sync(0xffffffffu, a0);
  const unsigned b1 = __ballot_sync(0xffffffffu, a1);
  if (a0) act[__popc(b0 & lt)] = lane;
  if (a1) act[__popc(b0) + __popc(b1 & lt)] = lane + 32;
  __syncwarp();
  return __popc(b0) + __popc(b1);
}

}  // namespace mova
