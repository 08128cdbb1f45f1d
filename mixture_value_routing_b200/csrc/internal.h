// Host-side launchers shared between the translation units of the library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mova.h"

namespace mova {

struct StatusBlock;

// Largest number of (token, slot) pairs the single-CTA grouping handles.
constexpr int kMaxPairs = 131072;
// Token counts up to this take the decode routing: a logits kernel over
// many CTAs, then selection and grouping by one CTA or inside the
// weight-streaming kernel.
constexpr int kFusedRouterMaxT = 8;

// Outputs of the grouping by expert (see launch_permute).
struct GroupOut {
  int32_t* counts;
  int32_t* offsets;
  int32_t* perm;
  int32_t* pos;
  int32_t* active;
  StatusBlock* sb;
  float* logits;     // decode routing: kMaxLogitSplits x 8 x 64 partial logits
};

// Router.  When g (with its logits scratch) is non-null and T <=
// kFusedRouterMaxT, the decode kernels also write the grouping (and *grouped
// is set); otherwise the caller runs launch_permute next.
// partitions: 1 (one fp32 sum per logit, any order) or 2 (the halves j < d/2
// and j >= d/2 summed separately in fp32, then added first + second).
cudaError_t launch_router(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                          int d, int E, int k, float scale, int32_t* idx, float* w,
                          const GroupOut* g, bool* grouped, int partitions, cudaStream_t stream);

// Decode routing in parts (T <= 8): the partial logits part[s][t][e] over S
// K ranges (S chosen here, returned in *S_out; at most 4), which also starts
// the call's status afresh; then selection and
// grouping by one CTA.  The weight-streaming kernel can take the place of
// the second part (RouteIn).
constexpr int kMaxLogitSplits = 4;
cudaError_t launch_router_logits(const void* x, mova_dtype x_dt, const float* Wr, int T, int d, int E,
                                 int partitions, float* part, int* S_out, StatusBlock* sb,
                                 cudaStream_t stream);
cudaError_t launch_select_group(const float* part, int S, const float* br, int T, int E, int k, float scale,
                                int32_t* idx, float* w, const GroupOut* g, cudaStream_t stream);
// The number S of K ranges the decode partial logits use.
int decode_logit_splits(int d, int E, int partitions);

// Every kernel launch the library enqueues is counted (mova_launch_count).
void note_launch();

// Launch with programmatic dependent launch enabled: the kernel may start
// while its predecessor on the stream finishes, and waits for it with
// griddepcontrol.wait before touching its outputs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  note_launch();
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Per-device SM count (cached).
int sm_count();

// cuTensorMapEncodeTiled from the driver (cached; nullptr if unavailable).
void* encode_tiled_fn();

// Tensor-core router (bf16 x): splits Wr into three bf16 planes (in
// `planes`, router_planes_bytes(d) bytes), then one CTA per 128 tokens
// computes the logits with tcgen05 and selects; tile_counts (nullable)
// receives each 128-token tile's expert histogram.
constexpr int kTcRouterMinT = 64;  // bf16 batches above this many tokens use it
size_t router_planes_bytes(int d);
// prepared: planes made by launch_split_router beforehand (then `planes` is
// not written), or null to split Wr into `planes` first.
cudaError_t launch_router_tc(const void* x, const float* Wr, const float* br, int T, int d, int E,
                             int k, float scale, int partitions, int32_t* idx, float* w,
                             int32_t* tile_counts, __nv_bfloat16* planes, const __nv_bfloat16* prepared,
                             StatusBlock* sb, cudaStream_t stream);
cudaError_t launch_split_router(const float* Wr, int E, int d, __nv_bfloat16* planes, cudaStream_t stream);

// Stable counting sort of the pairs by expert.  idx_in has dtype idx_dt
// (int32 or int8); when w_in is given (w_dt fp32 or fp16) it is converted to
// fp32 into w32, and idx_in to int32 into idx32 (routing-given mode).
cudaError_t launch_permute(const void* idx_in, mova_dtype idx_dt, const void* w_in,
                           mova_dtype w_dt, int N, int E, int32_t* idx32, float* w32,
                           int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                           int32_t* active, StatusBlock* sb, cudaStream_t stream);

// Multi-CTA grouping (batches above kSmallGroupT tokens).  Tiles of 128
// tokens; tile_counts holds group_tiles(T) x 64 ints.  launch_tile_hist
// fills tile_counts (and, in routing-given mode, idx32/w32 with the range
// check); launch_tile_group scans and scatters.
constexpr int kSmallGroupT = 512;
int group_tiles(int T);
cudaError_t launch_tile_hist(const void* idx_in, mova_dtype idx_dt, const void* w_in,
                             mova_dtype w_dt, int T, int E, int k, int32_t* idx32, float* w32,
                             int32_t* tile_counts, StatusBlock* sb, cudaStream_t stream);
cudaError_t launch_tile_group(const int32_t* idx32, int T, int E, int k, int32_t* tile_counts,
                              int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                              int32_t* active, StatusBlock* sb, bool reset_status, cudaStream_t stream);

// Weight-streaming expert kernel: P[p, :] = SiLU(Wv[e] x[t]) for every
// pair p (fp32 rows in grouped order).
// Routing done by the weight-streaming kernel itself (resident decode
// batches): every CTA sums the partial logits, selects and groups in shared
// memory; CTA 0 also writes idx_out / w_out.
struct RouteIn {
  const float* part;  // S x 8 x 64 partial logits (launch_router_logits); null: routing given
  int S;
  const float* br;
  int E;
  float scale;
  int32_t* idx_out;
  float* w_out;
  // The grouping CTA 0 computes (also written to global memory, so that it
  // can be read back from the workspace): counts (E), offsets (E+1), perm and
  // pos (T*k), the active list and the status block's active count.
  int32_t* counts_out;
  int32_t* offsets_out;
  int32_t* perm_out;
  int32_t* pos_out;
  int32_t* active_out;
  // One-launch decode (Wr non-null): the kernel first computes the partial
  // logits itself -- part[s][t][e] for the S K ranges, one (expert, range)
  // per CTA -- into part_out (== part), resets the status, and meets every other CTA at a grid barrier (slot bar_slot of
  // the library's ring of barrier words) before it selects.
  const float* Wr;
  float* part_out;
  int bar_slot;
};

// Ring of grid-barrier words of the one-launch decode kernel (library-owned
// device memory, zero at load, left as found by every completed barrier):
// the slot for the next launch, and a reset of the whole ring (after a
// barrier that ran out, which leaves its word unbalanced).
int next_grid_barrier_slot();
cudaError_t reset_grid_barriers(cudaStream_t stream);

// Test-only fault injection for the weight-streaming kernel
// (mova_selftest_arm_stream_stall): the limit of its pipeline waits in clock
// cycles, and the stage at which CTA 0's producer stops issuing weight
// copies (-1: never).  take_stream_fault() returns the armed values once and
// disarms them; unarmed it returns {kWaitLimitCycles, -1}.
struct StreamFault {
  long long wait_limit;
  int stall_stage;
  bool skip_barrier;  // the first CTA does not arrive at the one-launch grid barrier
};
StreamFault take_stream_fault();

// In resident mode (bf16, T <= 8; see stream_resident) v must be given and
// the kernel also performs the combine: each CTA owns a range of output
// columns and writes v there; the caller then skips launch_combine (P is not
// written).  Otherwise v is null.
// ldw: rows of Wv between consecutive experts' first rows (>= n).
cudaError_t launch_stream_experts(const void* x, const void* Wv, long long ldw, mova_dtype dt,
                                  const int32_t* counts,
                                  const int32_t* offsets, const int32_t* perm, const float* w32,
                                  const int32_t* active, StatusBlock* sb, int T, int d, int n,
                                  int k, int E, float* P, void* v, const RouteIn& route,
                                  cudaStream_t stream);

// Shared memory the streaming kernel needs for rows of d elements, n
// outputs per token and k of E experts per token (0 if d is too long for two
// 8-row stages).
size_t stream_experts_smem(int d, mova_dtype dt, int T, int n, int k, int E, int* stages_out);
// Whether the weight-streaming kernel keeps every token's x in shared memory
// for this batch (bf16, T <= 8, and its buffers fit; the mode in which it
// also performs the combine and may route: v must be given).  Otherwise the
// batch runs the per-chunk mode with a separate combine.
bool stream_resident(int T, int d, int n, int k, int E, mova_dtype dt);

// tcgen05 grouped GEMM (bf16): P[p, :] = SiLU(Wv[e] x[t]) as bf16 rows.
// xp: T*k x d bf16 scratch for the pairs' x rows in grouped order.
cudaError_t launch_tensor_experts(const void* x, const void* Wv, long long ldw, const int32_t* counts,
                                  const int32_t* offsets, const int32_t* pos, const float* w32,
                                  const int32_t* active, StatusBlock* sb, int T, int d, int n, int k,
                                  int E, __nv_bfloat16* xp, __nv_bfloat16* P, cudaStream_t stream);
size_t tensor_experts_smem();
// Attend mode of the pair GEMM (decode attention's PV product with V
// recomputed from the compact cache): probs (H, L) fp32, query head h reads
// KV head h / (H / (n / 128)), at most 4 query heads per KV head.  coef:
// L*k*(n/32) floats; part: attend_part_bytes; o: (H, 128) fp32.
size_t attend_part_bytes(int L, int E, int k, int n);
cudaError_t launch_tensor_attend(const void* Wv, const int32_t* counts, const int32_t* offsets,
                                 const int32_t* perm, const float* w32, StatusBlock* sb, int L, int d, int n,
                                 int k, int E, const float* probs, int H, const __nv_bfloat16* xp,
                                 float* coef, float* part, float* o, cudaStream_t stream);
// xp[pos[t * k + j]] = x[t] for the T*k pairs (token-major: each x row read once).
cudaError_t launch_gather_pairs(const void* x, const int32_t* pos, int T, int d, int k,
                                __nv_bfloat16* xp, cudaStream_t stream);
// The grouped GEMM on SM pairs (tcgen05 cta_group::2), reading the pairs'
// token rows already gathered into grouped order (xp, launch_gather_pairs);
// tiles of up to 512 pairs on two accumulators.
cudaError_t launch_tensor_experts_pair(const void* Wv, long long ldw, const int32_t* counts,
                                       const int32_t* offsets, StatusBlock* sb, int T,
                                       int d, int n, int k, int E, const __nv_bfloat16* xp, __nv_bfloat16* P,
                                       cudaStream_t stream);

// v[t, :] = sum over slots (ascending) of w[t*k + slot] * P[pos[t*k + slot], :].
cudaError_t launch_combine(const void* P, bool p_bf16, const int32_t* pos, const float* w32, int T,
                           int k, int n, void* v, mova_dtype v_dt, cudaStream_t stream);

}  // namespace mova
