// Permute: a stable counting sort of the T*k (token, rank) pairs by expert.
//
// Pairs are cut into chunks of CHUNK consecutive pair indices.
//   1. per-chunk histograms of the expert ids            (one CTA per chunk)
//   2. expert offsets = exclusive scan of the totals, and
//      base[c][e] = offsets[e] + sum_{c' < c} count[c'][e] (one CTA)
//   3. scatter: the CTA stages its chunk's ids in shared memory and cuts the
//      chunk into one run of consecutive pairs per warp; per-warp counts give
//      each warp its first row per expert (the chunk's base plus the counts
//      of the warps before it).  Each warp then walks its run 32 pairs at a
//      time; pairs of the same expert inside a step are ranked with
//      __match_any_sync, so a pair's row is its warp's base + (number of
//      earlier pairs of its expert).  No atomic decides any order, so the
//      result is deterministic.
// Small inputs (one chunk) run all three steps in a single CTA.
#include "sm100.cuh"

namespace ftmoe {

constexpr int kPermChunk = 1024;
constexpr int kMaxExperts = 1024;
constexpr int kScatterThreads = 256;

__device__ __forceinline__ bool valid_expert(int e, int E) { return e >= 0 && e < E; }

// Block-wide exclusive scan of one int per thread over blockDim.x <= 1024 threads.
__device__ int block_exclusive_scan(int v, int* smem_warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) smem_warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nwarps ? smem_warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, s, off);
      if (lane >= off) s += y;
    }
    if (lane < nwarps) smem_warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  const int before = warp > 0 ? smem_warp_sums[warp - 1] : 0;
  __syncthreads();
  return before + x - v;
}

// Walk pairs [p0, p1) in order with one warp; cursor[e] is this chunk's next
// row for expert e (shared memory), advanced as pairs are placed.  With
// SMEM_IDS the ids are read from a shared-memory copy indexed from p0 (the
// single-CTA path loads them once, in parallel, instead of one dependent
// global round trip per 32 pairs).
template <bool SMEM_IDS>
__device__ void scatter_chunk_warp(const int32_t* __restrict__ ids, int p0, int p1, int E, int* cursor,
                                   int32_t* __restrict__ perm_src, int32_t* __restrict__ pair_to_row,
                                   int P) {
  const int lane = threadIdx.x & 31;
  for (int base = p0; base < p1; base += 32) {
    const int p = base + lane;
    const bool live = p < p1;
    int e = live ? (SMEM_IDS ? ids[p - p0] : __ldg(ids + p)) : -1;
    if (live && !valid_expert(e, E)) { set_device_status(FT_DEV_BAD_INDEX); e = -1; }
    const uint32_t peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int leader = __ffs(peers) - 1;
    int row = -1;
    if (e >= 0) row = cursor[e] + rank;
    __syncwarp();
    if (e >= 0 && lane == leader) cursor[e] += __popc(peers);
    __syncwarp();
    if (e >= 0 && row >= 0 && row < P) {
      perm_src[row] = p;
      pair_to_row[p] = row;
    }
  }
}

// Whole permutation in one CTA (P <= kPermChunk).
__global__ void __launch_bounds__(1024) permute_small_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm_src,
                                                             int32_t* __restrict__ pair_to_row) {
  pdl_enter();
  __shared__ int cnt[kMaxExperts];
  __shared__ int warp_sums[32];
  __shared__ int32_t sids[kPermChunk];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < P; p += blockDim.x) {
    const int e = __ldg(ids + p);
    sids[p] = e;
    if (valid_expert(e, E)) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  // E <= 1024 = blockDim.x: one expert per thread
  const int e = threadIdx.x;
  const int c = e < E ? cnt[e] : 0;
  const int ex = block_exclusive_scan(c, warp_sums);
  if (e < E) { offsets[e] = ex; cnt[e] = ex; }
  if (e == E - 1) offsets[E] = ex + c;
  __syncthreads();
  if (threadIdx.x < 32) scatter_chunk_warp<true>(sids, 0, P, E, cnt, perm_src, pair_to_row, P);
}

__global__ void __launch_bounds__(256) permute_hist_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                           int32_t* __restrict__ counts) {
  pdl_enter();
  __shared__ int cnt[kMaxExperts];
  const int c = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  const int p0 = c * kPermChunk, p1 = min(P, p0 + kPermChunk);
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = __ldg(ids + p);
    if (valid_expert(e, E)) atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[size_t(c) * E + e] = cnt[e];
}

__global__ void __launch_bounds__(1024) permute_scan_kernel(int32_t* __restrict__ counts, int nchunks, int E,
                                                            int32_t* __restrict__ offsets) {
  pdl_enter();
  __shared__ int warp_sums[32];
  const int e = threadIdx.x;
  constexpr int kBatch = 8;   // loads in flight per thread
  int total = 0;
  if (e < E)
    for (int c0 = 0; c0 < nchunks; c0 += kBatch) {
      int n[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) n[i] = c0 + i < nchunks ? counts[size_t(c0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) total += n[i];
    }
  const int ex = block_exclusive_scan(total, warp_sums);
  if (e < E) {
    offsets[e] = ex;
    int run = ex;
    for (int c0 = 0; c0 < nchunks; c0 += kBatch) {  // counts become per-chunk base rows
      int n[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) n[i] = c0 + i < nchunks ? counts[size_t(c0 + i) * E + e] : 0;
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        if (c0 + i < nchunks) {
          counts[size_t(c0 + i) * E + e] = run;
          run += n[i];
        }
    }
  }
  if (e == E - 1) offsets[E] = ex + total;
}

__global__ void __launch_bounds__(kScatterThreads) permute_scatter_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                              const int32_t* __restrict__ bases,
                                                              int32_t* __restrict__ perm_src,
                                                              int32_t* __restrict__ pair_to_row) {
  pdl_enter();
  constexpr int kWarps = kScatterThreads / 32, kRun = kPermChunk / kWarps;
  __shared__ int32_t sids[kPermChunk];
  __shared__ int cursor[kWarps][kMaxExperts];   // per warp: its count, then its first row, per expert
  const int c = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = c * kPermChunk, p1 = min(P, p0 + kPermChunk);
  for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) cursor[i / E][i % E] = 0;
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) sids[p - p0] = __ldg(ids + p);
  __syncthreads();
  const int q0 = min(p1, p0 + warp * kRun), q1 = min(p1, q0 + kRun);   // this warp's run
  for (int p = q0 + lane; p < q1; p += 32) {
    const int e = sids[p - p0];
    if (valid_expert(e, E)) atomicAdd(&cursor[warp][e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = bases[size_t(c) * E + e];
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int n = cursor[w][e];
      cursor[w][e] = run;
      run += n;
    }
  }
  __syncthreads();
  if (q0 < q1) scatter_chunk_warp<true>(sids + (q0 - p0), q0, q1, E, cursor[warp], perm_src, pair_to_row, P);
}

// Route and permute in one CTA for small batches (T <= kFusedMaxT tokens,
// T*k <= kPermChunk pairs, E <= kFusedMaxE): each warp routes tokens with the
// same per-token code as route_kernel (so the same ids and weight bits), the
// selected ids stay in shared memory, and the counting sort of
// permute_small_kernel reads them from there.  Saves a launch and the ids'
// round trip through global memory on the decode path.
constexpr int kFusedMaxT = 128;
constexpr int kFusedMaxE = 512;

template <int NPL>
__global__ void __launch_bounds__(1024) route_permute_small_kernel(const float* __restrict__ logits, int T, int E,
                                                                   int k, int mode, int32_t* __restrict__ ids,
                                                                   float* __restrict__ wts,
                                                                   int32_t* __restrict__ offsets,
                                                                   int32_t* __restrict__ perm_src,
                                                                   int32_t* __restrict__ pair_to_row) {
  pdl_enter();
  __shared__ int s_ids[kPermChunk];
  __shared__ int cnt[kFusedMaxE];
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  for (int t = warp; t < T; t += nwarps) {
    int sel_id;
    float w;
    route_token<NPL>(logits + size_t(t) * E, E, k, mode, lane, sel_id, w);
    if (lane < k) {
      ids[size_t(t) * k + lane] = sel_id;
      wts[size_t(t) * k + lane] = w;
      s_ids[t * k + lane] = sel_id;
    }
  }
  __syncthreads();
  const int P = T * k;
  for (int p = threadIdx.x; p < P; p += blockDim.x) atomicAdd(&cnt[s_ids[p]], 1);
  __syncthreads();
  const int e = threadIdx.x;   // E <= kFusedMaxE <= blockDim.x: one expert per thread
  const int c = e < E ? cnt[e] : 0;
  const int ex = block_exclusive_scan(c, warp_sums);
  if (e < E) { offsets[e] = ex; cnt[e] = ex; }
  if (e == E - 1) offsets[E] = ex + c;
  __syncthreads();
  if (warp == 0) scatter_chunk_warp<true>(s_ids, 0, P, E, cnt, perm_src, pair_to_row, P);
}

static bool route_permute_fused_fits(int T, int k, int E) {
  return T >= 1 && T <= kFusedMaxT && T * k <= kPermChunk && E <= kFusedMaxE;
}

static cudaError_t launch_route_permute_small(const float* logits, int T, int E, int k, int mode, int32_t* ids,
                                              float* w, int32_t* offsets, int32_t* perm_src, int32_t* pair_to_row,
                                              cudaStream_t s) {
  const int npl = (E + 31) / 32;
  ProfileScope prof(FT_KERNEL_ROUTE_PERMUTE, s);
  auto kern = npl <= 1 ? route_permute_small_kernel<1> : npl <= 2 ? route_permute_small_kernel<2>
             : npl <= 4 ? route_permute_small_kernel<4> : npl <= 8 ? route_permute_small_kernel<8>
             : route_permute_small_kernel<16>;
  return launch_pdl(kern, dim3(1), dim3(1024), 0, s, logits, T, E, k, mode, ids, w, offsets, perm_src,
                    pair_to_row);
}

static size_t permute_ws_bytes(int T, int k, int E) {
  const long long P = (long long)T * k;
  const long long nchunks = (P + kPermChunk - 1) / kPermChunk;
  return nchunks <= 1 ? 0 : size_t(nchunks) * E * sizeof(int32_t);
}

static cudaError_t launch_permute(const int32_t* ids, int T, int k, int E, int32_t* offsets,
                                  int32_t* perm_src, int32_t* pair_to_row, void* ws, cudaStream_t s) {
  const int P = T * k;
  const int nchunks = (P + kPermChunk - 1) / kPermChunk;
  if (nchunks <= 1) {
    ProfileScope prof(FT_KERNEL_PERMUTE, s);
    return launch_pdl(permute_small_kernel, dim3(1), dim3(1024), 0, s, ids, P, E, offsets, perm_src, pair_to_row);
  }
  int32_t* counts = static_cast<int32_t*>(ws);
  cudaError_t e;
  {
    ProfileScope prof(FT_KERNEL_PERMUTE, s);
    e = launch_pdl(permute_hist_kernel, dim3(nchunks), dim3(256), 0, s, ids, P, E, counts);
  }
  if (e != cudaSuccess) return e;
  {
    ProfileScope prof(FT_KERNEL_PERMUTE, s);
    e = launch_pdl(permute_scan_kernel, dim3(1), dim3(1024), 0, s, counts, nchunks, E, offsets);
  }
  if (e != cudaSuccess) return e;
  ProfileScope prof(FT_KERNEL_PERMUTE, s);
  return launch_pdl(permute_scatter_kernel, dim3(nchunks), dim3(kScatterThreads), 0, s, ids, P, E,
                    static_cast<const int32_t*>(counts), perm_src, pair_to_row);
}

}  // namespace ftmoe
