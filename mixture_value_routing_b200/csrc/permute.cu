// Grouping of the (token, slot) pairs by expert: a stable counting sort.
//
// The expert mixture of "MoVA: routing the value vectors, and why the KV cache
// does not notice" (section "So what does it cost?") visits every touched
// expert once with the tokens routed to it.  Here the pairs f = t*k + slot
// are ordered by (expert, f): histogram, exclusive scan over experts, then a
// stable scatter.  No global atomics decide an order, so perm and pos are
// bit-exact and identical run to run.
//
// One CTA of 32 warps does the whole sort for up to 131072 pairs: each warp
// owns a contiguous segment of pairs, counts it into its own shared-memory
// histogram row, the rows are scanned per expert across warps (segment
// order), and each warp then ranks its segment 32 pairs at a time with
// __match_any_sync (rank = number of earlier lanes with the same expert).
// The expert codes are staged in shared memory as bytes between passes.
#include "common.cuh"
#include "internal.h"

namespace mova {

namespace {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;

template <typename IT, typename WT>
__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const IT* __restrict__ idx_in, const WT* __restrict__ w_in, int N, int E,
               int32_t* __restrict__ idx32, float* __restrict__ w32, int32_t* __restrict__ counts,
               int32_t* __restrict__ offsets, int32_t* __restrict__ perm, int32_t* __restrict__ pos,
               int32_t* __restrict__ active, StatusBlock* sb) {
  extern __shared__ uint8_t codes[];  // N expert codes
  __shared__ int hist[kPermWarps][64];
  __shared__ int tot[64];
  __shared__ int off[65];

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  for (int i = tid; i < kPermWarps * 64; i += kPermThreads) (&hist[0][0])[i] = 0;
  // The grouping is the first kernel of every value call that can raise a
  // device-side check: it starts the call's status afresh.
  if (tid == 0) {
    sb->code = 0;
    sb->detail = 0;
    sb->work_next = 0;
  }
  __syncthreads();

  const int seg = (N + kPermWarps - 1) / kPermWarps;
  const int f_begin = min(N, warp * seg);
  const int f_end = min(N, f_begin + seg);

  // Pass 1: read, check and stage the codes; per-warp histograms.
  for (int f = f_begin + lane; f < f_end; f += 32) {
    int e = static_cast<int>(idx_in[f]);
    if (e < 0 || e >= E) {
      raise_status(sb, MOVA_ERR_DEVICE_CHECK, f);
      e = 0;
    }
    codes[f] = static_cast<uint8_t>(e);
    if (idx32 != nullptr) idx32[f] = e;
    if (w32 != nullptr) w32[f] = to_f32(w_in[f]);
    atomicAdd(&hist[warp][e], 1);
  }
  __syncthreads();

  // Totals per expert, then the exclusive scan over experts.
  if (tid < 64) {
    int s = 0;
    for (int w = 0; w < kPermWarps; ++w) s += hist[w][tid];
    tot[tid] = (tid < E) ? s : 0;
  }
  __syncthreads();
  if (tid == 0) {
    int s = 0;
    for (int e = 0; e < E; ++e) {
      off[e] = s;
      s += tot[e];
    }
    off[E] = s;
  }
  __syncthreads();
  // hist[w][e] becomes the first position of warp w's pairs of expert e.
  if (tid < E) {
    int s = off[tid];
    for (int w = 0; w < kPermWarps; ++w) {
      const int c = hist[w][tid];
      hist[w][tid] = s;
      s += c;
    }
  }
  __syncthreads();

  // Pass 2: stable ranking inside each warp segment, in pair order.
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int c0 = f_begin; c0 < f_end; c0 += 32) {
    const int f = c0 + lane;
    const bool valid = f < f_end;
    const int e = valid ? static_cast<int>(codes[f]) : 0;
    const int key = valid ? e : 256 + lane;  // idle lanes form singleton groups
    const unsigned grp = __match_any_sync(0xffffffffu, key);
    const int rank = __popc(grp & lt_mask);
    const int size = __popc(grp);
    if (valid) {
      const int p = hist[warp][e] + rank;
      perm[p] = f;
      pos[f] = p;
    }
    __syncwarp();
    if (valid && rank == size - 1) hist[warp][e] += size;
    __syncwarp();
  }

  if (tid < E) {
    counts[tid] = tot[tid];
    offsets[tid] = off[tid];
  }
  if (tid == 0) offsets[E] = off[E];
  if (warp == 0) {
    const int e0 = lane, e1 = lane + 32;
    const bool a0 = e0 < E && tot[e0] > 0;
    const bool a1 = e1 < E && tot[e1] > 0;
    const unsigned m0 = __ballot_sync(0xffffffffu, a0);
    const unsigned m1 = __ballot_sync(0xffffffffu, a1);
    const int n0 = __popc(m0);
    if (a0) active[__popc(m0 & lt_mask)] = e0;
    if (a1) active[n0 + __popc(m1 & lt_mask)] = e1;
    if (lane == 0) sb->num_active = n0 + __popc(m1);
  }
}

template <typename IT, typename WT>
cudaError_t launch_t(const void* idx_in, const void* w_in, int N, int E, int32_t* idx32, float* w32,
                     int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                     int32_t* active, StatusBlock* sb, cudaStream_t stream) {
  auto kern = permute_kernel<IT, WT>;
  const size_t smem = static_cast<size_t>(N);
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kMaxPairs));
  if (err != cudaSuccess) return err;
  note_launch();
  kern<<<1, kPermThreads, smem, stream>>>(static_cast<const IT*>(idx_in),
                                          static_cast<const WT*>(w_in), N, E, idx32, w32, counts,
                                          offsets, perm, pos, active, sb);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Multi-CTA grouping for large batches: per-tile histograms, one scan, a
// stable scatter per tile.  A tile is 128 tokens (128 * k pairs, in pair
// order), so the tile order is the pair order and the result is the same
// stable sort as above.
// ---------------------------------------------------------------------------

constexpr int kTileTok = 128;

// Histogram of each tile's pairs; in routing-given mode also the int32 / fp32
// copies of the routing and the range check.
template <typename IT, typename WT>
__global__ void __launch_bounds__(256)
tile_hist_kernel(const IT* __restrict__ idx_in, const WT* __restrict__ w_in, int N, int E, int k,
                 int32_t* __restrict__ idx32, float* __restrict__ w32,
                 int32_t* __restrict__ tile_counts, StatusBlock* sb) {
  __shared__ int hist[64];
  if (threadIdx.x < 64) hist[threadIdx.x] = 0;
  __syncthreads();
  const int per = kTileTok * k;
  const int f0 = blockIdx.x * per;
  const int f1 = min(N, f0 + per);
  for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) {
    int e = static_cast<int>(idx_in[f]);
    if (e < 0 || e >= E) {
      raise_status(sb, MOVA_ERR_DEVICE_CHECK, f);
      e = 0;
    }
    if (idx32 != nullptr) idx32[f] = e;
    if (w32 != nullptr) w32[f] = to_f32(w_in[f]);
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  if (threadIdx.x < 64) tile_counts[blockIdx.x * 64 + threadIdx.x] = hist[threadIdx.x];
}

// Stable scatter of one tile.  Each CTA first derives, from every tile's
// histogram, the expert totals, their exclusive prefix (the expert offsets)
// and the number of its expert's pairs in earlier tiles, i.e. the first
// grouped position of each of its experts (CTA 0 also writes counts,
// offsets, the active list and the status fields).  Then 4 warps own
// consecutive segments of the tile's pairs; per-warp histograms are scanned
// in warp order on top of those positions, and each warp ranks 32 pairs at a
// time (earlier lanes with the same expert come first).
__global__ void __launch_bounds__(128)
tile_scatter_kernel(const int32_t* __restrict__ idx32, int N, int k, int E,
                    const int32_t* __restrict__ tile_counts, int ntiles, int32_t* __restrict__ counts,
                    int32_t* __restrict__ offsets, int32_t* __restrict__ active, StatusBlock* sb,
                    bool reset_status, int32_t* __restrict__ perm, int32_t* __restrict__ pos) {
  pdl_wait();
  __shared__ int hist[4][64];
  __shared__ int base[64];
  __shared__ int tot_s[64];
  __shared__ unsigned amask[2];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 4 * 64; i += 128) (&hist[0][0])[i] = 0;
  const unsigned lt_mask = (1u << lane) - 1u;
  if (threadIdx.x < 64) {
    // Thread e: the expert's total and its count in the tiles before this one.
    const int e = threadIdx.x;
    int tot = 0, before = 0;
    if (e < E) {
      for (int t = 0; t < ntiles; ++t) {
        const int c = tile_counts[t * 64 + e];
        tot += c;
        before += (t < static_cast<int>(blockIdx.x)) ? c : 0;
      }
    }
    // Exclusive prefix of the totals over experts (two warps).
    int inc = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    tot_s[e] = inc;  // inclusive within the warp
    const unsigned am = __ballot_sync(0xffffffffu, e < E && tot > 0);
    if (lane == 0) amask[warp] = am;
    asm volatile("bar.sync 1, 64;" ::: "memory");  // the two scanning warps
    const int warp0_total = tot_s[31];
    const int off = inc - tot + (warp == 1 ? warp0_total : 0);
    base[e] = off + before;
    if (blockIdx.x == 0) {
      if (e < E) {
        counts[e] = tot;
        offsets[e] = off;
      }
      if (e == E - 1) offsets[E] = off + tot;
      const int nbefore = (warp == 1) ? __popc(amask[0]) : 0;
      if (e < E && tot > 0) active[nbefore + __popc(am & lt_mask)] = e;
      if (e == 0) {
        if (reset_status) {
          sb->code = 0;
          sb->detail = 0;
        }
        sb->num_active = __popc(amask[0]) + __popc(amask[1]);
        sb->work_next = 0;
      }
    }
  }
  __syncthreads();
  const int per = kTileTok * k;
  const int t0 = blockIdx.x * per;
  const int t1 = min(N, t0 + per);
  const int seg = (per + 3) / 4;
  const int f_begin = min(t1, t0 + warp * seg);
  const int f_end = min(t1, f_begin + seg);
  for (int f = f_begin + lane; f < f_end; f += 32) atomicAdd(&hist[warp][idx32[f]], 1);
  __syncthreads();
  if (threadIdx.x < 64) {
    int b = base[threadIdx.x];
    for (int w = 0; w < 4; ++w) {
      const int c = hist[w][threadIdx.x];
      hist[w][threadIdx.x] = b;
      b += c;
    }
  }
  __syncthreads();
  for (int c0 = f_begin; c0 < f_end; c0 += 32) {
    const int f = c0 + lane;
    const bool valid = f < f_end;
    const int e = valid ? idx32[f] : 0;
    const unsigned grp = __match_any_sync(0xffffffffu, valid ? e : 256 + lane);
    const int rank = __popc(grp & lt_mask);
    const int size = __popc(grp);
    if (valid) {
      const int p = hist[warp][e] + rank;
      perm[p] = f;
      pos[f] = p;
    }
    __syncwarp();
    if (valid && rank == size - 1) hist[warp][e] += size;
    __syncwarp();
  }
}

template <typename IT, typename WT>
cudaError_t launch_hist_t(const void* idx_in, const void* w_in, int N, int E, int k, int32_t* idx32,
                          float* w32, int32_t* tile_counts, StatusBlock* sb, cudaStream_t stream) {
  const int ntiles = (N + kTileTok * k - 1) / (kTileTok * k);
  note_launch();
  tile_hist_kernel<IT, WT><<<ntiles, 256, 0, stream>>>(static_cast<const IT*>(idx_in),
                                                       static_cast<const WT*>(w_in), N, E, k, idx32,
                                                       w32, tile_counts, sb);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_permute(const void* idx_in, mova_dtype idx_dt, const void* w_in,
                           mova_dtype w_dt, int N, int E, int32_t* idx32, float* w32,
                           int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                           int32_t* active, StatusBlock* sb, cudaStream_t stream) {
  if (N <= 0 || N > kMaxPairs) return cudaErrorInvalidValue;
  if (w_in == nullptr) w32 = nullptr;
  if (idx_dt == MOVA_I8) {
    if (w_dt == MOVA_F16)
      return launch_t<int8_t, __half>(idx_in, w_in, N, E, idx32, w32, counts, offsets, perm, pos,
                                      active, sb, stream);
    return launch_t<int8_t, float>(idx_in, w_in, N, E, idx32, w32, counts, offsets, perm, pos,
                                   active, sb, stream);
  }
  if (w_dt == MOVA_F16)
    return launch_t<int32_t, __half>(idx_in, w_in, N, E, idx32, w32, counts, offsets, perm, pos,
                                     active, sb, stream);
  return launch_t<int32_t, float>(idx_in, w_in, N, E, idx32, w32, counts, offsets, perm, pos,
                                  active, sb, stream);
}

}  // namespace mova

namespace mova {

int group_tiles(int T) { return (T + kTileTok - 1) / kTileTok; }

cudaError_t launch_tile_hist(const void* idx_in, mova_dtype idx_dt, const void* w_in,
                             mova_dtype w_dt, int T, int E, int k, int32_t* idx32, float* w32,
                             int32_t* tile_counts, StatusBlock* sb, cudaStream_t stream) {
  const int N = T * k;
  if (w_in == nullptr) w32 = nullptr;
  // The status word is reset by the first kernel of the call that may raise it.
  cudaError_t err = cudaMemsetAsync(sb, 0, 8, stream);
  if (err != cudaSuccess) return err;
  if (idx_dt == MOVA_I8) {
    return w_dt == MOVA_F16
               ? launch_hist_t<int8_t, __half>(idx_in, w_in, N, E, k, idx32, w32, tile_counts, sb, stream)
               : launch_hist_t<int8_t, float>(idx_in, w_in, N, E, k, idx32, w32, tile_counts, sb, stream);
  }
  return w_dt == MOVA_F16
             ? launch_hist_t<int32_t, __half>(idx_in, w_in, N, E, k, idx32, w32, tile_counts, sb, stream)
             : launch_hist_t<int32_t, float>(idx_in, w_in, N, E, k, idx32, w32, tile_counts, sb, stream);
}

cudaError_t launch_tile_group(const int32_t* idx32, int T, int E, int k, int32_t* tile_counts,
                              int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                              int32_t* active, StatusBlock* sb, bool reset_status, cudaStream_t stream) {
  const int N = T * k;
  const int ntiles = group_tiles(T);
  return launch_pdl(tile_scatter_kernel, dim3(ntiles), dim3(128), 0, stream, idx32, N, k, E,
                    static_cast<const int32_t*>(tile_counts), ntiles, counts, offsets, active, sb,
                    reset_status, perm, pos);
}

}  // namespace mova
