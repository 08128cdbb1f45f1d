// C ABI entry points of the MoVA value path: argument checks, workspace
// layout, and the enqueueing of the kernels on the caller's stream.
//
// Call sequence of mova_value_routed (the pages' forward, "MoVA: routing the
// value vectors, and why the KV cache does not notice", section "Where the
// routing happens"):
//   router  -> idx, w                     (fp32 logits, sigmoid, biased top-k)
//   permute -> counts, offsets, perm, pos (stable grouping by expert)
//   experts -> P rows = SiLU(Wv[e] x)     (weight streaming or tcgen05 GEMM)
//   combine -> v = sum of w x row over each token's slots, ascending
#include <atomic>
#include <stdio.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace mova {

void* encode_tiled_fn() {
  static void* fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = p;
  }
  return fn;
}

namespace {
std::atomic<unsigned long long> g_launches{0};
// Armed by mova_selftest_arm_stream_stall for the next weight-streaming launch.
std::atomic<int> g_fault_stage{-1};
std::atomic<long long> g_fault_limit{0};
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

StreamFault take_stream_fault() {
  const int stage = g_fault_stage.exchange(-1);
  const long long limit = g_fault_limit.exchange(0);
  if (stage == -1 || limit <= 0) return StreamFault{kWaitLimitCycles, -1, false};
  if (stage == MOVA_STALL_AT_BARRIER) return StreamFault{limit, -1, true};
  return StreamFault{limit, stage, false};
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      sms = 148;
    cached[dev] = sms;
  }
  return cached[dev];
}

namespace {

// AUTO: bf16 batches above this many tokens use the tcgen05 grouped GEMM.
constexpr int kStreamMaxTokens = 64;
// bf16 batches up to this many tokens run the combine inside the
// weight-streaming kernel (the x rows stay resident there).
constexpr int kFusedCombineMaxT = 8;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Workspace {
  StatusBlock* sb;
  int32_t* idx;
  float* w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* active;
  int32_t* perm;
  int32_t* pos;
  float* logits;
  int32_t* tile_counts;
  __nv_bfloat16* planes;
  __nv_bfloat16* xp;
  void* P;
  size_t bytes;
};

// Byte layout of the workspace (every part 256-byte aligned).
Workspace layout(void* base, int T, int d, int k, int n) {
  const size_t pairs = static_cast<size_t>(T) * k;
  char* b = static_cast<char*>(base);
  size_t o = 0;
  Workspace w{};
  w.sb = reinterpret_cast<StatusBlock*>(b + o);       o += 256;
  w.idx = reinterpret_cast<int32_t*>(b + o);          o += align256(pairs * 4);
  w.w = reinterpret_cast<float*>(b + o);              o += align256(pairs * 4);
  w.counts = reinterpret_cast<int32_t*>(b + o);       o += 256;
  w.offsets = reinterpret_cast<int32_t*>(b + o);      o += 512;
  w.active = reinterpret_cast<int32_t*>(b + o);       o += 256;
  w.perm = reinterpret_cast<int32_t*>(b + o);         o += align256(pairs * 4);
  w.pos = reinterpret_cast<int32_t*>(b + o);          o += align256(pairs * 4);
  w.tile_counts = reinterpret_cast<int32_t*>(b + o);  o += align256(static_cast<size_t>(group_tiles(T)) * 64 * 4);
  w.planes = reinterpret_cast<__nv_bfloat16*>(b + o); o += align256(router_planes_bytes(d));
  // The decode partial logits (T <= 8, kMaxLogitSplits x 8 x 64 floats <= 192 * d * 2 bytes for
  // d >= 64) share the router planes' bytes: the planes exist only for T > 64.
  w.logits = reinterpret_cast<float*>(w.planes);
  w.xp = reinterpret_cast<__nv_bfloat16*>(b + o);     o += align256(pairs * static_cast<size_t>(d) * 2);
  w.P = b + o;                                        o += align256(pairs * static_cast<size_t>(n) * 4);
  w.bytes = o;
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

mova_status check_dims(int T, int d, int E, int k, int n) {
  if (T < 0 || d <= 0 || E <= 0 || k <= 0 || n <= 0) return MOVA_ERR_INVALID_ARG;
  if (k > E) return MOVA_ERR_INVALID_ARG;
  if (E > 64 || k > 8 || d % 64 != 0 || n % 128 != 0) return MOVA_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k > kMaxPairs) return MOVA_ERR_UNSUPPORTED;
  return MOVA_OK;
}

mova_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOVA_OK;
  fprintf(stderr, "mova: CUDA error %s\n", cudaGetErrorString(e));
  return MOVA_ERR_CUDA;
}

bool valid_act_dtype(mova_dtype dt) { return dt == MOVA_F32 || dt == MOVA_BF16; }

// Options with their defaults filled in.
struct Opts {
  mova_path path = MOVA_PATH_AUTO;
  void* const* events = nullptr;
  long long ldw = 0;   // rows between experts in Wv (n if 0 was given)
  int partitions = 1;  // router reduction halves (1 or 2)
  int decode_launches = 2;
  const void* planes = nullptr;  // prepared router planes
};

mova_status read_opts(const mova_options* o, int d, int n, Opts* out) {
  Opts r;
  if (o != nullptr) {
    r.path = o->path;
    r.events = o->events;
    r.ldw = o->wv_expert_stride;
    r.partitions = o->router_partitions == 0 ? 1 : o->router_partitions;
    r.decode_launches = o->decode_launches == 0 ? 2 : o->decode_launches;
    r.planes = o->router_planes;
  }
  if (r.planes != nullptr && (reinterpret_cast<uintptr_t>(r.planes) & 15) != 0) return MOVA_ERR_INVALID_ARG;
  if (r.decode_launches != 1 && r.decode_launches != 2) return MOVA_ERR_INVALID_ARG;
  if (r.path != MOVA_PATH_AUTO && r.path != MOVA_PATH_STREAM && r.path != MOVA_PATH_TENSOR &&
      r.path != MOVA_PATH_TENSOR_1CTA)
    return MOVA_ERR_INVALID_ARG;
  if (r.ldw == 0) r.ldw = n;
  if (r.ldw < n || r.ldw > (1LL << 24)) return MOVA_ERR_INVALID_ARG;
  if (r.partitions < 0) return MOVA_ERR_INVALID_ARG;
  if (r.partitions > 2 || (r.partitions == 2 && d % 128 != 0)) return MOVA_ERR_UNSUPPORTED;
  *out = r;
  return MOVA_OK;
}

// Records stage event i (if events were given); external so that it also
// becomes an event node under stream capture.
cudaError_t mark(void* const* events, int i, cudaStream_t s) {
  if (events == nullptr || events[i] == nullptr) return cudaSuccess;
  return cudaEventRecordWithFlags(static_cast<cudaEvent_t>(events[i]), s, cudaEventRecordExternal);
}

// Experts and combine, shared by both value entry points.
mova_status run_experts_and_combine(const void* x, mova_dtype dt, const void* Wv, long long ldw,
                                    const Workspace& ws, const int32_t* idx, const float* w32,
                                    int T, int d, int E, int k, int n, void* v, mova_path path,
                                    void* const* events, cudaStream_t stream) {
  (void)idx;
  if (path == MOVA_PATH_AUTO) path = mova_auto_path(T, dt);
  cudaError_t err = cudaSuccess;
  bool fused_combine = false;
  const bool tensor = path == MOVA_PATH_TENSOR || path == MOVA_PATH_TENSOR_1CTA;
  if (tensor && dt != MOVA_BF16) return MOVA_ERR_UNSUPPORTED;
  const bool pair = tensor && path == MOVA_PATH_TENSOR && sm_count() >= 2;
  // The pair GEMM's token rows are gathered first; the gather belongs to the
  // grouping stage, so the expert stage times the GEMM alone.
  if (pair) err = launch_gather_pairs(x, ws.pos, T, d, k, ws.xp, stream);
  if (err == cudaSuccess) err = mark(events, 2, stream);
  if (err != cudaSuccess) return from_cuda(err);
  if (tensor) {
    if (pair) {
      err = launch_tensor_experts_pair(Wv, ldw, ws.counts, ws.offsets, ws.sb, T, d, n, k, E, ws.xp,
                                       static_cast<__nv_bfloat16*>(ws.P), stream);
    } else {
      err = launch_tensor_experts(x, Wv, ldw, ws.counts, ws.offsets, ws.pos, w32, ws.active, ws.sb, T,
                                  d, n, k, E, ws.xp, static_cast<__nv_bfloat16*>(ws.P), stream);
    }
  } else {
    if (stream_experts_smem(d, dt, T, n, k, E, nullptr) == 0) return MOVA_ERR_UNSUPPORTED;
    // Decode-sized bf16 batches fold the combine into the expert kernel.
    fused_combine = T <= kFusedCombineMaxT && stream_resident(T, d, n, k, E, dt);
    err = launch_stream_experts(x, Wv, ldw, dt, ws.counts, ws.offsets, ws.perm, w32, ws.active, ws.sb,
                                T, d, n, k, E, static_cast<float*>(ws.P),
                                fused_combine ? v : nullptr,
                                RouteIn{}, stream);
  }
  if (err == cudaSuccess) err = mark(events, 3, stream);
  if (err == cudaSuccess && !fused_combine)
    err = launch_combine(ws.P, tensor, ws.pos, w32, T, k, n, v, dt, stream);
  if (err == cudaSuccess) err = mark(events, 4, stream);
  return from_cuda(err);
}

// Self-test of the bounded waits: one thread waits on an mbarrier that
// nothing will ever arrive at, gives up after `limit` cycles and reports
// MOVA_ERR_TIMEOUT in the status block, as every pipeline wait does.
__global__ void selftest_wait_kernel(StatusBlock* sb, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sb->code = 0;
    sb->detail = 0;
    mbar_init(&bar, 1);
    fence_barrier_init();
    if (!mbar_wait_for(&bar, 0, limit)) raise_status(sb, MOVA_ERR_TIMEOUT, 1);
  }
}

}  // namespace
}  // namespace mova

using namespace mova;

extern "C" {

const char* mova_status_str(mova_status s) {
  switch (s) {
    case MOVA_OK: return "MOVA_OK";
    case MOVA_ERR_INVALID_ARG: return "MOVA_ERR_INVALID_ARG";
    case MOVA_ERR_UNSUPPORTED: return "MOVA_ERR_UNSUPPORTED";
    case MOVA_ERR_CUDA: return "MOVA_ERR_CUDA";
    case MOVA_ERR_TIMEOUT: return "MOVA_ERR_TIMEOUT";
    case MOVA_ERR_DEVICE_CHECK: return "MOVA_ERR_DEVICE_CHECK";
  }
  return "MOVA_ERR_UNKNOWN";
}

size_t mova_workspace_size(int T, int d, int E, int k, int n) {
  if (check_dims(T, d, E, k, n) != MOVA_OK) return 0;
  if (T == 0) return 0;
  return layout(nullptr, T, d, k, n).bytes;
}

unsigned long long mova_launch_count(void) { return mova::g_launches.load(); }

// Attend mode: the value workspace plus the per-group partials.
static bool attend_heads_ok(int n, int H) {
  const int nkv = n / 128;
  return H > 0 && nkv > 0 && H % nkv == 0 && H / nkv <= 4;
}

size_t mova_attend_workspace_size(int L, int d, int E, int k, int n, int H) {
  if (check_dims(L, d, E, k, n) != MOVA_OK || !attend_heads_ok(n, H) || L == 0) return 0;
  return layout(nullptr, L, d, k, n).bytes + align256(attend_part_bytes(L, E, k, n));
}

mova_status mova_value_attend(const void* x, const void* idx, mova_dtype idx_dt, const void* wgt,
                              mova_dtype w_dt, const void* Wv, int L, int d, int E, int k, int n,
                              const float* probs, int H, float* o, void* ws, size_t ws_bytes, void* stream) {
  mova_status st = check_dims(L, d, E, k, n);
  if (st != MOVA_OK) return st;
  if (H <= 0) return MOVA_ERR_INVALID_ARG;
  if (!attend_heads_ok(n, H)) return MOVA_ERR_UNSUPPORTED;
  if (idx_dt != MOVA_I32 && idx_dt != MOVA_I8) return MOVA_ERR_UNSUPPORTED;
  if (w_dt != MOVA_F32 && w_dt != MOVA_F16) return MOVA_ERR_UNSUPPORTED;
  if (!o) return MOVA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (L == 0) return from_cuda(cudaMemsetAsync(o, 0, static_cast<size_t>(H) * 128 * sizeof(float), s));
  if (!x || !idx || !wgt || !Wv || !probs || !ws) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wv)) return MOVA_ERR_INVALID_ARG;
  if (sm_count() < 2) return MOVA_ERR_UNSUPPORTED;  // the pair GEMM
  const Workspace w = layout(ws, L, d, k, n);
  const size_t part_off = w.bytes;
  if (ws_bytes < part_off + align256(attend_part_bytes(L, E, k, n)) || (reinterpret_cast<uintptr_t>(ws) & 255) != 0)
    return MOVA_ERR_INVALID_ARG;
  cudaError_t err;
  if (L > kSmallGroupT) {
    err = launch_tile_hist(idx, idx_dt, wgt, w_dt, L, E, k, w.idx, w.w, w.tile_counts, w.sb, s);
    if (err == cudaSuccess)
      err = launch_tile_group(w.idx, L, E, k, w.tile_counts, w.counts, w.offsets, w.perm, w.pos, w.active, w.sb,
                              false, s);
  } else {
    err = launch_permute(idx, idx_dt, wgt, w_dt, L * k, E, w.idx, w.w, w.counts, w.offsets, w.perm, w.pos,
                         w.active, w.sb, s);
  }
  if (err == cudaSuccess) err = launch_gather_pairs(x, w.pos, L, d, k, w.xp, s);
  if (err == cudaSuccess)
    err = launch_tensor_attend(Wv, w.counts, w.offsets, w.perm, w.w, w.sb, L, d, n, k, E, probs, H, w.xp,
                               static_cast<float*>(w.P),
                               reinterpret_cast<float*>(static_cast<char*>(ws) + part_off), o, s);
  return from_cuda(err);
}

mova_path mova_auto_path(int T, mova_dtype x_dt) {
  return (x_dt == MOVA_BF16 && T > kStreamMaxTokens) ? MOVA_PATH_TENSOR : MOVA_PATH_STREAM;
}

mova_status mova_route_opts(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                            int d, int E, int k, float scale, int32_t* idx, float* w,
                            const mova_options* opts, void* stream) {
  mova_status st = check_dims(T, d, E, k, 128);
  if (st != MOVA_OK) return st;
  Opts o;
  st = read_opts(opts, d, 128, &o);
  if (st != MOVA_OK) return st;
  if (!valid_act_dtype(x_dt)) return MOVA_ERR_UNSUPPORTED;
  if (T == 0) return MOVA_OK;
  if (!x || !Wr || !br || !idx || !w) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wr)) return MOVA_ERR_INVALID_ARG;
  return from_cuda(launch_router(x, x_dt, Wr, br, T, d, E, k, scale, idx, w, nullptr, nullptr,
                                 o.partitions, static_cast<cudaStream_t>(stream)));
}

size_t mova_router_planes_bytes(int d) { return d > 0 && d % 64 == 0 ? router_planes_bytes(d) : 0; }

mova_status mova_router_planes(const float* Wr, int E, int d, void* planes, void* stream) {
  if (!Wr || !planes || E < 1 || E > 64 || d <= 0 || d % 64 != 0) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(Wr) || !aligned16(planes)) return MOVA_ERR_INVALID_ARG;
  return from_cuda(launch_split_router(Wr, E, d, static_cast<__nv_bfloat16*>(planes),
                                       static_cast<cudaStream_t>(stream)));
}

mova_status mova_route(const void* x, mova_dtype x_dt, const float* Wr, const float* br, int T,
                       int d, int E, int k, float scale, int32_t* idx, float* w, void* stream) {
  return mova_route_opts(x, x_dt, Wr, br, T, d, E, k, scale, idx, w, nullptr, stream);
}

mova_status mova_permute(const int32_t* idx, int T, int E, int k, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* pos, void* ws, size_t ws_bytes,
                         void* stream) {
  mova_status st = check_dims(T, 64, E, k, 128);
  if (st != MOVA_OK) return st;
  if (T == 0) return MOVA_OK;
  if (!idx || !counts || !offsets || !perm || !pos || !ws) return MOVA_ERR_INVALID_ARG;
  const Workspace w = layout(ws, T, 64, k, 128);
  if (ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOVA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (T > kSmallGroupT) {
    cudaError_t err = launch_tile_hist(idx, MOVA_I32, nullptr, MOVA_F32, T, E, k, nullptr, nullptr,
                                       w.tile_counts, w.sb, s);
    if (err == cudaSuccess)
      err = launch_tile_group(idx, T, E, k, w.tile_counts, counts, offsets, perm, pos, w.active, w.sb,
                              false, s);
    return from_cuda(err);
  }
  return from_cuda(launch_permute(idx, MOVA_I32, nullptr, MOVA_F32, T * k, E, nullptr, nullptr,
                                  counts, offsets, perm, pos, w.active, w.sb, s));
}

mova_status mova_value_opts(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                            const void* wgt, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt, int T,
                            int d, int E, int k, int n, void* v, void* ws, size_t ws_bytes,
                            const mova_options* opts, void* stream) {
  mova_status st = check_dims(T, d, E, k, n);
  if (st != MOVA_OK) return st;
  Opts o;
  st = read_opts(opts, d, n, &o);
  if (st != MOVA_OK) return st;
  const mova_path path = o.path;
  void* const* events = o.events;
  if (!valid_act_dtype(x_dt) || wv_dt != x_dt) return MOVA_ERR_UNSUPPORTED;
  if ((path == MOVA_PATH_TENSOR || path == MOVA_PATH_TENSOR_1CTA) && x_dt != MOVA_BF16)
    return MOVA_ERR_UNSUPPORTED;  // the tensor-core kernels take bf16 only
  if (idx_dt != MOVA_I32 && idx_dt != MOVA_I8) return MOVA_ERR_UNSUPPORTED;
  if (w_dt != MOVA_F32 && w_dt != MOVA_F16) return MOVA_ERR_UNSUPPORTED;
  if (T == 0) return MOVA_OK;
  if (!x || !idx || !wgt || !Wv || !v || !ws) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wv) || !aligned16(v)) return MOVA_ERR_INVALID_ARG;
  if ((o.ldw * d * (x_dt == MOVA_BF16 ? 2 : 4)) % 16 != 0) return MOVA_ERR_INVALID_ARG;
  const Workspace w = layout(ws, T, d, k, n);
  if (ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOVA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = mark(events, 0, s);
  if (err == cudaSuccess) err = mark(events, 1, s);
  if (err == cudaSuccess) {
    if (T > kSmallGroupT) {
      err = launch_tile_hist(idx, idx_dt, wgt, w_dt, T, E, k, w.idx, w.w, w.tile_counts, w.sb, s);
      if (err == cudaSuccess)
        err = launch_tile_group(w.idx, T, E, k, w.tile_counts, w.counts, w.offsets, w.perm, w.pos,
                                w.active, w.sb, false, s);
    } else {
      err = launch_permute(idx, idx_dt, wgt, w_dt, T * k, E, w.idx, w.w, w.counts, w.offsets, w.perm,
                           w.pos, w.active, w.sb, s);
    }
  }
  if (err != cudaSuccess) return from_cuda(err);
  return run_experts_and_combine(x, x_dt, Wv, o.ldw, w, w.idx, w.w, T, d, E, k, n, v, path, events, s);
}

mova_status mova_value_ex(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                          const void* wgt, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt, int T,
                          int d, int E, int k, int n, void* v, void* ws, size_t ws_bytes,
                          mova_path path, void* const* events, void* stream) {
  const mova_options o{path, events, 0, 0, 0, nullptr};
  return mova_value_opts(x, x_dt, idx, idx_dt, wgt, w_dt, Wv, wv_dt, T, d, E, k, n, v, ws, ws_bytes, &o,
                         stream);
}

mova_status mova_value(const void* x, mova_dtype x_dt, const void* idx, mova_dtype idx_dt,
                       const void* wgt, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt, int T,
                       int d, int E, int k, int n, void* v, void* ws, size_t ws_bytes,
                       void* stream) {
  return mova_value_ex(x, x_dt, idx, idx_dt, wgt, w_dt, Wv, wv_dt, T, d, E, k, n, v, ws, ws_bytes,
                       MOVA_PATH_AUTO, nullptr, stream);
}

mova_status mova_value_routed_opts(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                                   const void* Wv, mova_dtype wv_dt, int T, int d, int E, int k,
                                   int n, float scale, void* v, int32_t* idx_out, float* w_out,
                                   void* ws, size_t ws_bytes, const mova_options* opts,
                                   void* stream) {
  mova_status st = check_dims(T, d, E, k, n);
  if (st != MOVA_OK) return st;
  Opts o;
  st = read_opts(opts, d, n, &o);
  if (st != MOVA_OK) return st;
  const mova_path path = o.path;
  void* const* events = o.events;
  if (!valid_act_dtype(x_dt) || wv_dt != x_dt) return MOVA_ERR_UNSUPPORTED;
  if ((path == MOVA_PATH_TENSOR || path == MOVA_PATH_TENSOR_1CTA) && x_dt != MOVA_BF16)
    return MOVA_ERR_UNSUPPORTED;  // the tensor-core kernels take bf16 only
  if (T == 0) return MOVA_OK;
  if (!x || !Wr || !br || !Wv || !v || !ws) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(Wr) || !aligned16(Wv) || !aligned16(v))
    return MOVA_ERR_INVALID_ARG;
  if ((o.ldw * d * (x_dt == MOVA_BF16 ? 2 : 4)) % 16 != 0) return MOVA_ERR_INVALID_ARG;
  const Workspace w = layout(ws, T, d, k, n);
  if (ws_bytes < w.bytes || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOVA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* idx = idx_out ? idx_out : w.idx;
  float* wgt = w_out ? w_out : w.w;
  const GroupOut g{w.counts, w.offsets, w.perm, w.pos, w.active, w.sb, w.logits};
  bool grouped = false;
  cudaError_t err = mark(events, 0, s);
  // Decode batches on the weight-streaming path: the router computes the
  // logits only; the streaming kernel selects, groups and combines.
  const mova_path rp = path == MOVA_PATH_AUTO ? mova_auto_path(T, x_dt) : path;
  if (rp == MOVA_PATH_STREAM && T <= kFusedCombineMaxT && stream_resident(T, d, n, k, E, x_dt) &&
      stream_experts_smem(d, x_dt, T, n, k, E, nullptr) != 0) {
    int S = 0;
    const bool one = o.decode_launches == 1;
    if (one) {
      S = decode_logit_splits(d, E, o.partitions);
    } else if (err == cudaSuccess) {
      err = launch_router_logits(x, x_dt, Wr, T, d, E, o.partitions, w.logits, &S, w.sb, s);
    }
    if (err == cudaSuccess) err = mark(events, 1, s);
    if (err == cudaSuccess) err = mark(events, 2, s);
    const RouteIn ri{w.logits, S,       br,         E,        scale,   idx,   wgt,
                     w.counts, w.offsets, w.perm, w.pos, w.active,
                     one ? Wr : nullptr, w.logits, one ? next_grid_barrier_slot() : 0};
    if (err == cudaSuccess)
      err = launch_stream_experts(x, Wv, o.ldw, x_dt, w.counts, w.offsets, w.perm, wgt, w.active, w.sb, T, d,
                                  n, k, E, static_cast<float*>(w.P), v, ri, s);
    if (err == cudaSuccess) err = mark(events, 3, s);
    if (err == cudaSuccess) err = mark(events, 4, s);
    return from_cuda(err);
  }
  // bf16 batches above the decode range route on the tensor cores and group
  // with the tile kernels (the router writes the per-tile histograms).
  const bool tc_router = x_dt == MOVA_BF16 && T > kTcRouterMinT;
  if (err == cudaSuccess) {
    if (tc_router)
      err = launch_router_tc(x, Wr, br, T, d, E, k, scale, o.partitions, idx, wgt, w.tile_counts, w.planes,
                             static_cast<const __nv_bfloat16*>(o.planes), w.sb, s);
    else
      err = launch_router(x, x_dt, Wr, br, T, d, E, k, scale, idx, wgt, &g, &grouped, o.partitions, s);
  }
  if (err == cudaSuccess) err = mark(events, 1, s);
  if (err == cudaSuccess && !grouped) {
    if (tc_router) {
      err = launch_tile_group(idx, T, E, k, w.tile_counts, w.counts, w.offsets, w.perm, w.pos, w.active,
                              w.sb, true, s);
    } else if (T > kSmallGroupT) {
      err = launch_tile_hist(idx, MOVA_I32, nullptr, MOVA_F32, T, E, k, nullptr, nullptr, w.tile_counts,
                             w.sb, s);
      if (err == cudaSuccess)
        err = launch_tile_group(idx, T, E, k, w.tile_counts, w.counts, w.offsets, w.perm, w.pos,
                                w.active, w.sb, false, s);
    } else {
      err = launch_permute(idx, MOVA_I32, nullptr, MOVA_F32, T * k, E, nullptr, nullptr, w.counts,
                           w.offsets, w.perm, w.pos, w.active, w.sb, s);
    }
  }
  if (err != cudaSuccess) return from_cuda(err);
  return run_experts_and_combine(x, x_dt, Wv, o.ldw, w, idx, wgt, T, d, E, k, n, v, path, events, s);
}

mova_status mova_value_routed_ex(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                                 const void* Wv, mova_dtype wv_dt, int T, int d, int E, int k,
                                 int n, float scale, void* v, int32_t* idx_out, float* w_out,
                                 void* ws, size_t ws_bytes, mova_path path, void* const* events,
                                 void* stream) {
  const mova_options o{path, events, 0, 0, 0, nullptr};
  return mova_value_routed_opts(x, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v, idx_out, w_out, ws,
                                ws_bytes, &o, stream);
}

mova_status mova_value_routed(const void* x, mova_dtype x_dt, const float* Wr, const float* br,
                              const void* Wv, mova_dtype wv_dt, int T, int d, int E, int k, int n,
                              float scale, void* v, int32_t* idx_out, float* w_out, void* ws,
                              size_t ws_bytes, void* stream) {
  return mova_value_routed_ex(x, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v, idx_out, w_out,
                              ws, ws_bytes, MOVA_PATH_AUTO, nullptr, stream);
}

mova_status mova_selftest_wait_timeout(void* ws, long long limit_cycles, void* stream) {
  if (!ws || limit_cycles <= 0 || limit_cycles > kWaitLimitCycles) return MOVA_ERR_INVALID_ARG;
  note_launch();
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<StatusBlock*>(ws), limit_cycles);
  return from_cuda(cudaGetLastError());
}

mova_status mova_selftest_arm_stream_stall(int stall_stage, long long limit_cycles) {
  if ((stall_stage < 0 && stall_stage != MOVA_STALL_AT_BARRIER) || limit_cycles <= 0 ||
      limit_cycles > kWaitLimitCycles)
    return MOVA_ERR_INVALID_ARG;
  g_fault_limit.store(limit_cycles);
  g_fault_stage.store(stall_stage);
  return MOVA_OK;
}

mova_status mova_workspace_parts(int T, int d, int E, int k, int n, size_t* offsets) {
  if (offsets == nullptr) return MOVA_ERR_INVALID_ARG;
  const mova_status st = check_dims(T, d, E, k, n);
  if (st != MOVA_OK) return st;
  if (T == 0) return MOVA_ERR_INVALID_ARG;
  const Workspace w = layout(nullptr, T, d, k, n);
  const void* parts[MOVA_WS_PARTS] = {w.idx, w.w, w.counts, w.offsets, w.perm, w.pos};
  for (int i = 0; i < MOVA_WS_PARTS; ++i) offsets[i] = reinterpret_cast<uintptr_t>(parts[i]);
  return MOVA_OK;
}

// ---- Host-buffer forms ------------------------------------------------------
// The batch's inputs are copied from host memory into staging space that
// follows the device call's workspace, the device call runs on it, and the
// result is copied back to host memory: three steps on the caller's stream.

static size_t act_size(mova_dtype dt) { return dt == MOVA_BF16 ? 2 : 4; }
static size_t idx_size(mova_dtype dt) { return dt == MOVA_I8 ? 1 : 4; }
static size_t wgt_size(mova_dtype dt) { return dt == MOVA_F16 ? 2 : 4; }

// Staging of a value call: x (at most 4 B an element), v, idx and w.
static size_t value_staging_bytes(int T, int d, int k, int n) {
  const size_t Tz = static_cast<size_t>(T);
  return align256(Tz * d * 4) + align256(Tz * n * 4) + 2 * align256(Tz * k * 4);
}

size_t mova_workspace_size_host(int T, int d, int E, int k, int n) {
  const size_t base = mova_workspace_size(T, d, E, k, n);
  if (base == 0) return 0;
  return align256(base) + value_staging_bytes(T, d, k, n);
}

static bool host_ws_ok(const void* ws, size_t ws_bytes, size_t need) {
  return need != 0 && ws_bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255) == 0;
}

// The one support condition the device call checks only on its chosen path:
// the weight-streaming kernel's shared memory for this d.  Checked here
// first, so that nothing is enqueued when the call would be refused.
static bool host_path_supported(int T, int d, int E, int k, int n, mova_dtype dt) {
  return mova_auto_path(T, dt) != MOVA_PATH_STREAM || stream_experts_smem(d, dt, T, n, k, E, nullptr) != 0;
}

mova_status mova_value_routed_host(const void* x_host, mova_dtype x_dt, const float* Wr, const float* br,
                                   const void* Wv, mova_dtype wv_dt, int T, int d, int E, int k, int n,
                                   float scale, void* v_host, int32_t* idx_host, float* w_host, void* ws,
                                   size_t ws_bytes, void* stream) {
  mova_status st = check_dims(T, d, E, k, n);
  if (st != MOVA_OK) return st;
  if (!valid_act_dtype(x_dt) || wv_dt != x_dt) return MOVA_ERR_UNSUPPORTED;
  if (T == 0) return MOVA_OK;
  if (!x_host || !Wr || !br || !Wv || !v_host || !ws) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(Wr) || !aligned16(Wv)) return MOVA_ERR_INVALID_ARG;
  if (!host_ws_ok(ws, ws_bytes, mova_workspace_size_host(T, d, E, k, n))) return MOVA_ERR_INVALID_ARG;
  if (!host_path_supported(T, d, E, k, n, x_dt)) return MOVA_ERR_UNSUPPORTED;
  const size_t base = align256(mova_workspace_size(T, d, E, k, n));
  const size_t Tz = static_cast<size_t>(T), es = act_size(x_dt);
  char* x_dev = static_cast<char*>(ws) + base;
  char* v_dev = x_dev + align256(Tz * d * 4);
  int32_t* idx_dev = reinterpret_cast<int32_t*>(v_dev + align256(Tz * n * 4));
  float* w_dev = reinterpret_cast<float*>(reinterpret_cast<char*>(idx_dev) + align256(Tz * k * 4));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemcpyAsync(x_dev, x_host, Tz * d * es, cudaMemcpyHostToDevice, s);
  if (err != cudaSuccess) return from_cuda(err);
  st = mova_value_routed(x_dev, x_dt, Wr, br, Wv, wv_dt, T, d, E, k, n, scale, v_dev,
                         idx_host ? idx_dev : nullptr, w_host ? w_dev : nullptr, ws, base, stream);
  if (st != MOVA_OK) return st;
  err = cudaMemcpyAsync(v_host, v_dev, Tz * n * es, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess && idx_host) err = cudaMemcpyAsync(idx_host, idx_dev, Tz * k * 4, cudaMemcpyDeviceToHost, s);
  if (err == cudaSuccess && w_host) err = cudaMemcpyAsync(w_host, w_dev, Tz * k * 4, cudaMemcpyDeviceToHost, s);
  return from_cuda(err);
}

mova_status mova_value_host(const void* x_host, mova_dtype x_dt, const void* idx_host, mova_dtype idx_dt,
                            const void* w_host, mova_dtype w_dt, const void* Wv, mova_dtype wv_dt, int T, int d,
                            int E, int k, int n, void* v_host, void* ws, size_t ws_bytes, void* stream) {
  mova_status st = check_dims(T, d, E, k, n);
  if (st != MOVA_OK) return st;
  if (!valid_act_dtype(x_dt) || wv_dt != x_dt) return MOVA_ERR_UNSUPPORTED;
  if (idx_dt != MOVA_I32 && idx_dt != MOVA_I8) return MOVA_ERR_UNSUPPORTED;
  if (w_dt != MOVA_F32 && w_dt != MOVA_F16) return MOVA_ERR_UNSUPPORTED;
  if (T == 0) return MOVA_OK;
  if (!x_host || !idx_host || !w_host || !Wv || !v_host || !ws) return MOVA_ERR_INVALID_ARG;
  if (!aligned16(Wv)) return MOVA_ERR_INVALID_ARG;
  if (!host_ws_ok(ws, ws_bytes, mova_workspace_size_host(T, d, E, k, n))) return MOVA_ERR_INVALID_ARG;
  if (!host_path_supported(T, d, E, k, n, x_dt)) return MOVA_ERR_UNSUPPORTED;
  const size_t base = align256(mova_workspace_size(T, d, E, k, n));
  const size_t Tz = static_cast<size_t>(T), es = act_size(x_dt);
  char* x_dev = static_cast<char*>(ws) + base;
  char* v_dev = x_dev + align256(Tz * d * 4);
  char* idx_dev = v_dev + align256(Tz * n * 4);
  char* w_dev = idx_dev + align256(Tz * k * 4);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaMemcpyAsync(x_dev, x_host, Tz * d * es, cudaMemcpyHostToDevice, s);
  if (err == cudaSuccess)
    err = cudaMemcpyAsync(idx_dev, idx_host, Tz * k * idx_size(idx_dt), cudaMemcpyHostToDevice, s);
  if (err == cudaSuccess) err = cudaMemcpyAsync(w_dev, w_host, Tz * k * wgt_size(w_dt), cudaMemcpyHostToDevice, s);
  if (err != cudaSuccess) return from_cuda(err);
  st = mova_value(x_dev, x_dt, idx_dev, idx_dt, w_dev, w_dt, Wv, wv_dt, T, d, E, k, n, v_dev, ws, base, stream);
  if (st != MOVA_OK) return st;
  return from_cuda(cudaMemcpyAsync(v_host, v_dev, Tz * n * es, cudaMemcpyDeviceToHost, s));
}

// Staging of an attend call: x (bf16), idx and w (at most 4 B), probs, o.
static size_t attend_staging_bytes(int L, int d, int k, int H) {
  const size_t Lz = static_cast<size_t>(L);
  return align256(Lz * d * 2) + 2 * align256(Lz * k * 4) + align256(static_cast<size_t>(H) * Lz * 4) +
         align256(static_cast<size_t>(H) * 128 * 4);
}

size_t mova_attend_workspace_size_host(int L, int d, int E, int k, int n, int H) {
  if (check_dims(L, d, E, k, n) != MOVA_OK || !attend_heads_ok(n, H)) return 0;
  return align256(mova_attend_workspace_size(L, d, E, k, n, H)) + attend_staging_bytes(L, d, k, H);
}

mova_status mova_value_attend_host(const void* x_host, const void* idx_host, mova_dtype idx_dt,
                                   const void* w_host, mova_dtype w_dt, const void* Wv, int L, int d, int E,
                                   int k, int n, const float* probs_host, int H, float* o_host, void* ws,
                                   size_t ws_bytes, void* stream) {
  mova_status st = check_dims(L, d, E, k, n);
  if (st != MOVA_OK) return st;
  if (H <= 0) return MOVA_ERR_INVALID_ARG;
  if (!attend_heads_ok(n, H)) return MOVA_ERR_UNSUPPORTED;
  if (idx_dt != MOVA_I32 && idx_dt != MOVA_I8) return MOVA_ERR_UNSUPPORTED;
  if (w_dt != MOVA_F32 && w_dt != MOVA_F16) return MOVA_ERR_UNSUPPORTED;
  if (!o_host || !ws) return MOVA_ERR_INVALID_ARG;
  if (L > 0 && (!x_host || !idx_host || !w_host || !Wv || !probs_host)) return MOVA_ERR_INVALID_ARG;
  if (L > 0 && !aligned16(Wv)) return MOVA_ERR_INVALID_ARG;
  if (L > 0 && sm_count() < 2) return MOVA_ERR_UNSUPPORTED;  // the pair GEMM
  if (!host_ws_ok(ws, ws_bytes, mova_attend_workspace_size_host(L, d, E, k, n, H))) return MOVA_ERR_INVALID_ARG;
  const size_t base = align256(mova_attend_workspace_size(L, d, E, k, n, H));
  const size_t Lz = static_cast<size_t>(L), Hz = static_cast<size_t>(H);
  char* x_dev = static_cast<char*>(ws) + base;
  char* idx_dev = x_dev + align256(Lz * d * 2);
  char* w_dev = idx_dev + align256(Lz * k * 4);
  float* p_dev = reinterpret_cast<float*>(w_dev + align256(Lz * k * 4));
  float* o_dev = reinterpret_cast<float*>(reinterpret_cast<char*>(p_dev) + align256(Hz * Lz * 4));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  if (L > 0) {
    err = cudaMemcpyAsync(x_dev, x_host, Lz * d * 2, cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(idx_dev, idx_host, Lz * k * idx_size(idx_dt), cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess) err = cudaMemcpyAsync(w_dev, w_host, Lz * k * wgt_size(w_dt), cudaMemcpyHostToDevice, s);
    if (err == cudaSuccess) err = cudaMemcpyAsync(p_dev, probs_host, Hz * Lz * 4, cudaMemcpyHostToDevice, s);
    if (err != cudaSuccess) return from_cuda(err);
  }
  st = mova_value_attend(x_dev, idx_dev, idx_dt, w_dev, w_dt, Wv, L, d, E, k, n, p_dev, H, o_dev, ws, base,
                         stream);
  if (st != MOVA_OK) return st;
  return from_cuda(cudaMemcpyAsync(o_host, o_dev, Hz * 128 * 4, cudaMemcpyDeviceToHost, s));
}

mova_status mova_get_status(void* ws, int32_t* detail_out, void* stream) {
  if (!ws) return MOVA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return from_cuda(err);
  StatusBlock sb{};
  err = cudaMemcpy(&sb, ws, sizeof(sb), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return from_cuda(err);
  if (detail_out) *detail_out = sb.detail;
  if (sb.code == MOVA_ERR_TIMEOUT) {
    // A grid barrier that ran out leaves its word unbalanced: restore the ring.
    err = reset_grid_barriers(s);
    if (err == cudaSuccess) err = cudaStreamSynchronize(s);
    if (err != cudaSuccess) return from_cuda(err);
  }
  return static_cast<mova_status>(sb.code);
}

}  // extern "C"
