/*
 * mova.h -- C ABI of the MoVA value path on NVIDIA B200 (sm_100a).
 *
 * MoVA (Mixture-of-Value Attention) replaces an attention layer's GQA value
 * projection by a router over E value experts, each a full d -> n value
 * projection.  For every token t with hidden state x[t] (length d):
 *
 *   logits[t,e] = sum_j x[t,j] * Wr[e,j]          (router, no bias, fp32)
 *   s[t,e]      = sigmoid(logits[t,e])
 *   idx[t,:]    = the k experts with the largest s[t,e] + br[e]
 *                 (descending; equal scores -> lower expert index first)
 *   w[t,slot]   = scale * s[t,idx[t,slot]] / sum_slots s[t,idx[t,slot']]
 *   v[t,:]      = sum_{slot = 0..k-1, ascending} w[t,slot] * SiLU(Wv[idx[t,slot]] x[t])
 *
 * and v, of shape (T, n) = (T, heads, head_dim), is exactly the tensor a
 * GQA v_proj would have produced.  Source: "MoVA: routing the value vectors,
 * and why the KV cache does not notice" (ai.thesatyajit.com), section
 * "Where the routing happens" (router call, gate with the bias handed
 * separately, top-4, scale 2.5, SiLU mixture, reshape to 128-wide heads);
 * section "So what does it cost?" (64 experts of 2560 x 1024 per layer).
 * The routing-given entry point recomputes v from a stored x and its routing
 * as in the compact cache of "IFM K2 Horizon Deep Dive ...", Section 4,
 * Option B.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *    and contiguous, 16-byte aligned, except the batch and result buffers of
 *    the *_host entry points, which are HOST pointers.  The library never
 *    allocates.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every compute call is asynchronous on it; outputs are valid
 *    once the stream has reached that point.
 *  - Argument errors are detected on the host before anything is enqueued
 *    and returned synchronously; nothing is written then.
 *  - Errors that only the device can see (an expert index out of range in
 *    routing-given mode, a bounded wait that ran out) are recorded in a
 *    status word at the start of the workspace; read it with
 *    mova_get_status().  Offending entries are clamped so that no access
 *    leaves its buffer.
 *  - T == 0 is a valid no-op and returns MOVA_OK.
 *  - The weights (Wr, br, Wv and prepared router planes) are read as
 *    constants.  A call's first kernel may be chained to the kernel before
 *    it on the stream with programmatic dependent launch, and the router
 *    kernels start reading Wr and br before they wait for that kernel.
 *    Inputs and outputs (x, idx, w, v, the workspace) are touched only after
 *    the wait.  A caller that writes router weights with a kernel (an online
 *    bias update, say) must let it complete before the call: write them on
 *    another stream and make this one wait on an event recorded after the
 *    write, or synchronize.
 *  - Supported on the GPU: 1 <= E <= 64, 1 <= k <= min(E, 8), d % 64 == 0,
 *    n % 128 == 0, T * k <= 131072; dtypes x/Wv/v all fp32, or all bf16
 *    (router Wr/br always fp32).  The weight-streaming expert kernel also
 *    needs d <= 4608 (bf16) or d <= 3456 (fp32).  Anything else returns
 *    MOVA_ERR_UNSUPPORTED; there is no fallback path.
 */
#ifndef MOVA_H_
#define MOVA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOVA_OK = 0,
  MOVA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, workspace too small */
  MOVA_ERR_UNSUPPORTED = 2,   /* valid arguments the library does not implement */
  MOVA_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
  MOVA_ERR_TIMEOUT = 4,       /* a bounded device-side wait ran out (status word) */
  MOVA_ERR_DEVICE_CHECK = 5   /* a device-side input check failed (status word) */
} mova_status;

typedef enum {
  MOVA_F32 = 0,
  MOVA_BF16 = 1,
  MOVA_F16 = 2,
  MOVA_I32 = 3,
  MOVA_I8 = 4
} mova_dtype;

/* Which expert kernel runs.  AUTO picks the weight-streaming kernel for
 * small token counts (and for fp32) and the tcgen05 grouped GEMM on SM pairs
 * for bf16 batches above a threshold.  STREAM and TENSOR force one;
 * TENSOR_1CTA forces the single-CTA variant of the grouped GEMM (TENSOR*
 * require bf16; otherwise MOVA_ERR_UNSUPPORTED). */
typedef enum {
  MOVA_PATH_AUTO = 0,
  MOVA_PATH_STREAM = 1,
  MOVA_PATH_TENSOR = 2,
  MOVA_PATH_TENSOR_1CTA = 3
} mova_path;

/* Human-readable name of a status code (static storage, never NULL). */
const char* mova_status_str(mova_status s);

/* Bytes of device workspace the value entry points need for these sizes
 * (0 when T == 0).  The workspace holds the status word, the routing, the
 * grouping by expert and the per-(token, slot) expert outputs; it may be
 * reused across calls on the same stream.  Returns 0 for invalid sizes. */
size_t mova_workspace_size(int T, int d, int E, int k, int n);

/* Router: sigmoid gate, bias-assisted top-k, renormalise, scale.
 *   x    (T, d)  x_dt in {MOVA_F32, MOVA_BF16}
 *   Wr   (E, d)  fp32 router weight;  br (E) fp32 router bias (selection only)
 *   idx  (T, k)  int32 out: selected experts, slot 0 = highest biased score
 *   w    (T, k)  fp32 out: scale * s / sum(s) over the k selected
 * Logits are accumulated in fp32.  Source: "Where the routing happens". */
mova_status mova_route(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                       int T, int d, int E, int k, float scale,
                       int32_t* idx, float* w, void* stream);

/* Grouping of the flat (token, slot) pairs f = t*k + slot by expert: a
 * stable counting sort.
 *   idx     (T, k) int32 in [0, E)
 *   counts  (E)    int32 out: pairs per expert
 *   offsets (E+1)  int32 out: exclusive prefix sum of counts
 *   perm    (T*k)  int32 out: the pair at each position of the order sorted
 *                  by (expert, f)
 *   pos     (T*k)  int32 out: inverse of perm
 * Bit-exact and deterministic.  An index outside [0, E) is clamped and
 * raises MOVA_ERR_DEVICE_CHECK in the status word held by `ws`
 * (ws_bytes >= mova_workspace_size(T, 64, E, k, 128) suffices).
 * Source: "So what does it cost?" (the released combine visits each touched
 * expert once with its tokens; this is that grouping, made deterministic). */
mova_status mova_permute(const int32_t* idx, int T, int E, int k,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                         void* ws, size_t ws_bytes, void* stream);

/* Routing-given mixture (compact-cache recompute):
 *   v[t] = sum_{slot ascending} w[t,slot] * SiLU(Wv[idx[t,slot]] x[t])
 *   x   (T, d)    x_dt in {MOVA_F32, MOVA_BF16}
 *   idx (T, k)    idx_dt in {MOVA_I32, MOVA_I8}
 *   w   (T, k)    w_dt in {MOVA_F32, MOVA_F16}; used as given (no renormalisation)
 *   Wv  (E, n, d) wv_dt == x_dt; expert e's weight is output-major (n rows of d)
 *   v   (T, n)    same dtype as x; equals (T, n/128, 128) GQA value heads
 *   ws  device workspace of ws_bytes >= mova_workspace_size(T, d, E, k, n)
 * Source: "IFM K2 Horizon Deep Dive ...", Section 4, Option B (the cache
 * keeps x, the top-4 indices and fp16 weights; V is recomputed), with the
 * mixture of "Where the routing happens". */
mova_status mova_value(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                       const void* w, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt,
                       int T, int d, int E, int k, int n, void* v,
                       void* ws, size_t ws_bytes, void* stream);

/* Full value path: route, group, expert projections with SiLU x weight,
 * fixed-order combine.  Arguments as in mova_route and mova_value; idx_out
 * (T, k) int32 and w_out (T, k) fp32 are optional copies of the routing
 * (pass NULL to skip).  Source: "Where the routing happens" (the forward:
 * router, gate with the bias, top-4, scale 2.5, SiLU mixture, reshape to
 * 128-wide heads). */
mova_status mova_value_routed(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                              const void* Wv, mova_dtype wv_dt,
                              int T, int d, int E, int k, int n, float scale, void* v,
                              int32_t* idx_out, float* w_out,
                              void* ws, size_t ws_bytes, void* stream);

/* As mova_value / mova_value_routed, with the expert kernel chosen by
 * `path` instead of automatically, and optional stage timing: `events`
 * (nullable) points to MOVA_STAGE_EVENTS cudaEvent_t handles (passed as
 * void*, created by the caller) that are recorded on `stream` at the stage
 * boundaries: [0] start, [1] after routing, [2] after grouping, [3] after the
 * expert kernel, [4] after the combine (mova_value_ex records [0] and [1]
 * together, as its routing is given).  They are recorded with
 * cudaEventRecordExternal, so they also work inside CUDA graph capture. */
#define MOVA_STAGE_EVENTS 5
mova_status mova_value_ex(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                          const void* w, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt,
                          int T, int d, int E, int k, int n, void* v,
                          void* ws, size_t ws_bytes, mova_path path, void* const* events,
                          void* stream);
mova_status mova_value_routed_ex(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                                 const void* Wv, mova_dtype wv_dt,
                                 int T, int d, int E, int k, int n, float scale, void* v,
                                 int32_t* idx_out, float* w_out,
                                 void* ws, size_t ws_bytes, mova_path path, void* const* events,
                                 void* stream);

/* Where a value call leaves its routing and grouping inside the workspace.
 * Writes MOVA_WS_PARTS byte offsets, relative to the start of a workspace
 * laid out for these sizes, of:
 *   [0] idx     (T, k)  int32  the routing the expert kernels used, unless the
 *   [1] w       (T, k)  fp32   call wrote it to caller-given idx_out / w_out
 *   [2] counts  (E)     int32  pairs per expert
 *   [3] offsets (E+1)   int32  exclusive prefix sum of counts
 *   [4] perm    (T*k)   int32  pair f = t*k + slot at each grouped position
 *   [5] pos     (T*k)   int32  inverse of perm
 * (the arrays mova_permute defines).  Every value entry point fills [2]-[5]
 * with the grouping its expert kernels ran on, so a caller (or a test) can
 * read it back once the stream has passed the call.  Host-only; returns
 * MOVA_ERR_INVALID_ARG / MOVA_ERR_UNSUPPORTED as mova_workspace_size would
 * return 0, and for T == 0 (no workspace). */
#define MOVA_WS_PARTS 6
mova_status mova_workspace_parts(int T, int d, int E, int k, int n, size_t* offsets);

/* Options of the _opts entry points (zero-initialise, then set what is
 * needed; a NULL options pointer means all defaults).
 *
 *  path, events       as for mova_value_ex / mova_value_routed_ex.
 *
 *  wv_expert_stride   rows of Wv from one expert's first row to the next
 *                     expert's (0 means n: the dense (E, n, d) layout).  With
 *                     a stride the call reads only rows [0, n) of each
 *                     expert, so a head-parallel rank computes its slice of
 *                     the value heads straight from a full (E, n_total, d)
 *                     tensor: pass Wv + row0 * d, n = its rows, stride =
 *                     n_total.  v then holds that rank's (T, n) slice, i.e.
 *                     its n / 128 heads.  This is the tensor-parallel serving
 *                     layout of "IFM/K2-Horizon-MoVA-36B-A4B" (paperfeed.app),
 *                     "What's actually there, and maturity" (2 GPUs, TP = 2):
 *                     the router is replicated, every rank routes the same
 *                     tokens identically, and no collective is needed because
 *                     the heads stay on their rank.  Must be >= n (else
 *                     MOVA_ERR_INVALID_ARG); the start of every expert's rows
 *                     must stay 16-byte aligned.
 *
 *  router_partitions  0 or 1: each logit is one fp32 sum over d, in an order
 *                     the kernels choose.  2: the router's reduction over d
 *                     runs as two halves, j < d/2 and j >= d/2, each summed in
 *                     fp32, and the two fp32 partial sums are then added
 *                     (first + second).  This reproduces a router GEMM split
 *                     into two K partitions, the setting the serving recipes
 *                     pass to keep a checkpoint's router numerics
 *                     ("xllm_source_router_gemm_partitions: 2";
 *                     "Mixture of Value Attention" (robotsatlas.com),
 *                     "Implementation pitfalls").  Where partial sums cancel,
 *                     the rounding of each half to fp32 decides the logit, and
 *                     so the selection.  Needs d % 128 == 0; other values
 *                     return MOVA_ERR_UNSUPPORTED.
 *
 *  decode_launches    bf16 decode batches (T <= 8) on the weight-streaming
 *                     path.  1: one persistent kernel per call -- every CTA
 *                     first computes part of the router logits, all CTAs
 *                     meet at a grid barrier (bounded wait), then each
 *                     selects, groups, streams its share of the active
 *                     experts' weights and combines.  0 or 2 (the default,
 *                     measured 0.7 us faster per T = 8 step on B200, as the
 *                     logits kernel overlaps the previous call's tail): the
 *                     logits in a kernel of their own, then the streaming
 *                     kernel (chained with programmatic dependent launch).
 *                     Both give identical results.
 *
 *  router_planes      NULL, or the router weight already split by
 *                     mova_router_planes (for this Wr, E and d): bf16 batches
 *                     routed on the tensor cores (T > 64) then skip the split
 *                     of every call.  The planes depend on Wr only, so a
 *                     model makes them once per layer when it loads.
 *
 *                     The barrier words
 *                     are library-owned device memory, a ring of 64 reused
 *                     in turn, so calls on one stream never share one; calls
 *                     in flight at once on different streams of one device
 *                     may, when 64 or more are, and must then use 2.  The one
 *                     kernel needs all its CTAs (one per SM) resident at
 *                     once: with the device shared by other work a call may
 *                     report MOVA_ERR_TIMEOUT instead; use 2 there. */
typedef struct mova_options {
  mova_path path;
  void* const* events;
  long long wv_expert_stride;
  int router_partitions;
  int decode_launches;
  const void* router_planes;
} mova_options;

/* The fp32 router weight Wr (E, d) split exactly into three bf16 planes,
 * Wr = hi + mid + lo (each the round-to-nearest bf16 of what the previous
 * ones left; 8 + 8 + 8 significand bits cover fp32's 24), stored as a
 * (3 * 64, d) bf16 matrix: row e of plane p at row 64 * p + e, rows E..63 of
 * each plane zero.  The tensor-core router multiplies bf16 x by these planes,
 * forming every product exactly, and adds the three fp32 accumulations
 * (hi + mid) + lo: the logits of an fp32 dot product, accumulated in another
 * order.  `planes` (device, 16-byte aligned) receives
 * mova_router_planes_bytes(d) bytes; asynchronous on `stream`.  The routing
 * calls split Wr themselves unless mova_options.router_planes is given.
 * Errors: MOVA_ERR_INVALID_ARG for null or misaligned pointers, E outside
 * [1, 64] or d not a positive multiple of 64. */
size_t mova_router_planes_bytes(int d);
mova_status mova_router_planes(const float* Wr, int E, int d, void* planes, void* stream);

/* Decode attention's value side over the compact cache, with V never
 * written to memory ("IFM K2 Horizon Deep Dive", Section 4, Option B: the
 * cache keeps x, the top-k indices and the fp16 weights; V is rematerialised
 * on the fly inside the attention).  For L cached positions with hidden
 * states x (L, d) bf16, given routing idx (L, k) int8/int32 and weights
 * wgt (L, k) fp16/fp32, and attention probabilities probs (H, L) fp32 of one
 * query token's H heads:
 *
 *   o[h, :] = sum over l of probs[h, l] * V[l, h / G, :],   G = H / (n / 128)
 *
 * where V[l] = sum over slots (ascending) of w[l, slot] * SiLU(Wv[idx[l, slot]] x[l]),
 * viewed as (n / 128) KV heads of 128 ("MoVA: routing the value vectors",
 * section "Where the routing happens": the mixture is what a GQA v_proj
 * writes; query head h reads KV head h / G).  o: (H, 128) fp32, device.
 * bf16 x and Wv only; 1 <= G <= 4; runs the tensor-core expert kernel with
 * an epilogue that sums p * w * SiLU(h) per tile instead of storing V, then
 * a fixed-order reduction (results do not depend on timing).  Workspace:
 * mova_attend_workspace_size(L, d, E, k, n, H) bytes, 256-byte aligned.
 * L = 0 writes zeros.  Errors as mova_value; MOVA_ERR_UNSUPPORTED for H not a
 * multiple of n / 128 or G > 4. */
size_t mova_attend_workspace_size(int L, int d, int E, int k, int n, int H);
mova_status mova_value_attend(const void* x, const void* idx, mova_dtype idx_dt, const void* wgt,
                              mova_dtype w_dt, const void* Wv, int L, int d, int E, int k, int n,
                              const float* probs, int H, float* o, void* ws, size_t ws_bytes, void* stream);

/* Host-buffer forms of mova_value_routed, mova_value and mova_value_attend,
 * for callers whose batch lives in host memory.  The same computation and
 * arguments, except that the batch's inputs (x; idx and w of a given routing;
 * probs) are HOST pointers, read by cudaMemcpyAsync into staging space at the
 * end of the device workspace, and the result (v, or o; with
 * mova_value_routed_host also the optional idx_out / w_out copies of the
 * routing) is written to HOST memory by cudaMemcpyAsync.  The weights (Wr,
 * br, Wv) stay DEVICE pointers.  Order on `stream`: input copies, the device
 * call, output copies.
 *  - Host buffers: page-locked (cudaHostAlloc / pinned) memory makes both
 *    copies asynchronous; pageable memory works, with the driver's
 *    synchronous staging.  The caller keeps the inputs unchanged and does not
 *    read the outputs until the stream has passed the call (e.g. after
 *    cudaStreamSynchronize or an event).
 *  - Workspace: mova_workspace_size_host(T, d, E, k, n) bytes for the two
 *    value forms, mova_attend_workspace_size_host(L, d, E, k, n, H) for the
 *    attend form (also > 0 for L = 0, which writes zeros to o), 256-byte
 *    aligned device memory; the device call uses its first part, the staging
 *    the rest.  Two calls in flight on different streams need two workspaces.
 *  - Errors: as the device forms, all detected before anything is enqueued
 *    (a CUDA error from a copy returns MOVA_ERR_CUDA). */
size_t mova_workspace_size_host(int T, int d, int E, int k, int n);
size_t mova_attend_workspace_size_host(int L, int d, int E, int k, int n, int H);
mova_status mova_value_routed_host(const void* x_host, mova_dtype x_dt, const float* Wr, const float* br,
                                   const void* Wv, mova_dtype wv_dt, int T, int d, int E, int k, int n,
                                   float scale, void* v_host, int32_t* idx_host, float* w_host, void* ws,
                                   size_t ws_bytes, void* stream);
mova_status mova_value_host(const void* x_host, mova_dtype x_dt, const void* idx_host, mova_dtype idx_dt,
                            const void* w_host, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt, int T, int d,
                            int E, int k, int n, void* v_host, void* ws, size_t ws_bytes, void* stream);
mova_status mova_value_attend_host(const void* x_host, const void* idx_host, mova_dtype idx_dt,
                                   const void* w_host, mova_dtype w_dt, const void* Wv, int L, int d, int E,
                                   int k, int n, const float* probs_host, int H, float* o_host, void* ws,
                                   size_t ws_bytes, void* stream);

/* mova_route with options (only router_partitions applies). */
mova_status mova_route_opts(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                            int T, int d, int E, int k, float scale, int32_t* idx, float* w,
                            const mova_options* opts, void* stream);
/* mova_value with options (path, events, wv_expert_stride). */
mova_status mova_value_opts(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                            const void* w, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt,
                            int T, int d, int E, int k, int n, void* v,
                            void* ws, size_t ws_bytes, const mova_options* opts, void* stream);
/* mova_value_routed with options (all of them). */
mova_status mova_value_routed_opts(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                                   const void* Wv, mova_dtype wv_dt,
                                   int T, int d, int E, int k, int n, float scale, void* v,
                                   int32_t* idx_out, float* w_out,
                                   void* ws, size_t ws_bytes, const mova_options* opts, void* stream);

/* Synchronises `stream`, then returns and clears the device status word
 * held in `ws` (MOVA_OK if no device-side check fired since the last read).
 * `detail_out` (nullable) receives the first offending item (e.g. the flat
 * pair index of a bad expert index).  After a MOVA_ERR_TIMEOUT it also
 * restores the one-launch decode kernel's grid-barrier words, which a wait
 * that ran out leaves unbalanced. */
mova_status mova_get_status(void* ws, int32_t* detail_out, void* stream);

/* Self-test of the device-side failure detection: launches one thread that
 * waits on a barrier nothing arrives at, with the same bounded wait every
 * pipeline kernel uses but a limit of `limit_cycles` clock cycles (at most
 * about one second's worth); it then records MOVA_ERR_TIMEOUT in the status
 * word of `ws` (256 bytes suffice), readable with mova_get_status.  The
 * context stays usable afterwards.  Not part of the method. */
mova_status mova_selftest_wait_timeout(void* ws, long long limit_cycles, void* stream);

/* Self-test of the weight-streaming kernel's failure handling: arms the
 * next weight-streaming launch in this process so that its first CTA stops
 * issuing weight copies at stage `stall_stage` (>= 0), or -- with
 * MOVA_STALL_AT_BARRIER -- does not arrive at the one-launch decode kernel's
 * grid barrier; its waits give up after `limit_cycles` clock cycles (at most
 * about one second's worth).  That launch then records MOVA_ERR_TIMEOUT in
 * the status word, every warp leaves, the copies already issued are
 * drained, and the context stays usable (mova_get_status, reading that
 * timeout, also restores the barrier words).  The arming is consumed by that
 * one launch.  Not part of the method; returns MOVA_ERR_INVALID_ARG for
 * another negative stage or a limit out of range. */
#define MOVA_STALL_AT_BARRIER (-2)
mova_status mova_selftest_arm_stream_stall(int stall_stage, long long limit_cycles);

/* The path AUTO would pick for these sizes and dtype (for tests/benches). */
mova_path mova_auto_path(int T, mova_dtype x_dt);

/* Number of kernel launches this library has enqueued in this process so far
 * (all devices and threads; a launch enqueued into a stream capture counts
 * once, however often the graph is replayed).  The difference across a call
 * is the number of kernels that call issues.  Never fails. */
unsigned long long mova_launch_count(void);

/* Size of the workspace array built into the library for
 * mova_value_routed_noalloc. */
#define MOVA_NOALLOC_SCRATCH_BYTES (2u << 20)

/* mova_value_routed without a caller-provided workspace, for callers that
 * cannot allocate device memory where they run the value projection: code
 * inside a stream capture that must not add allocation nodes, programs whose
 * memory pool owns all of the device memory, or plug-ins that are handed only
 * the tensors they compute on.  (The MoVA pages have no counterpart: this is
 * a deployment convenience, not part of the method.)
 *
 * Arguments, layouts, results and errors are those of mova_value_routed
 * (automatic kernel choice, no routing copies).  The workspace is a
 * MOVA_NOALLOC_SCRATCH_BYTES array compiled into the library; every GPU that
 * loads the library holds it until the process exits.  Nothing is allocated
 * or freed: no cudaMalloc, cudaFree or allocating library routine is called.
 *  - Sizes whose mova_workspace_size exceeds MOVA_NOALLOC_SCRATCH_BYTES are
 *    rejected with MOVA_ERR_UNSUPPORTED (and a message on stderr); at
 *    d = 2560, E = 64, k = 4, n = 1024 that admits batches up to T = 30.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.  The address is kept per device and context
 *    (keyed on the context's process-unique id); after cudaDeviceReset, or
 *    with another context current, the next call looks it up again, so make
 *    that call outside a capture too.  If the driver cannot report context
 *    ids, every call looks the address up.
 *  - All calls share the one array and it keeps the last call's contents;
 *    each call's first kernel resets the status fields it relies on, and
 *    every other part is fully rewritten.  Calls on one device that may
 *    overlap on the GPU (calls on different streams) race: order them on one
 *    stream.  Each device holds its own copy of the array, so calls on
 *    different devices do not interfere.  The device status word is not
 *    exposed. */
mova_status mova_value_routed_noalloc(const void* x, mova_dtype x_dt, const float* Wr,
                                      const float* br, const void* Wv, mova_dtype wv_dt,
                                      int T, int d, int E, int k, int n, float scale, void* v,
                                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOVA_H_ */
