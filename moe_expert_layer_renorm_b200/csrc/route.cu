// Router: top-k over fp32 logits with renormalised weights.
//
// One warp per token.  Lane l holds logits l, l+32, l+64, ... in registers
// (coalesced loads).  k rounds of a warp argmax (largest value; equal values
// -> lower expert id) pick the experts in descending order, so the selected
// set and its order depend only on fp32 comparisons of the logits.  The
// weights are then computed in fp32:
//   FT_ROUTE_TOPK_SOFTMAX  : w_j = exp(l_j - m) / sum_S exp(l_i - m)
//   FT_ROUTE_SOFTMAX_RENORM: p_i = exp(l_i - m) / sum_all exp(l - m); w_j = p_j / sum_S p
// with m the largest logit (the two are one function up to rounding).
#include "sm100.cuh"

namespace ftmoe {

// The top-k and weights of one token, computed by one warp: lane j < k gets
// the j-th selected expert and its weight.  `row` points at the token's E
// logits.
template <int NPL>  // logits per lane = ceil(E / 32)
__device__ __forceinline__ void route_token(const float* __restrict__ row, int E, int k, int mode, int lane,
                                            int& sel_id_out, float& w_out) {
  float v[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = e < E ? __ldg(row + e) : 0.0f;
  }
  uint32_t taken = 0;  // bit i: entry i of this lane is selected (or absent)
#pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (lane + 32 * i >= E) taken |= 1u << i;

  float sel_v = 0.0f;  // lane j < k keeps the j-th selected logit and id
  int sel_id = 0;
  float vmax = 0.0f;
  for (int j = 0; j < k; ++j) {
    // local best among untaken entries; ascending i means ascending id
    float bv = 0.0f;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
      if (!(taken & (1u << i)) && (bi < 0 || v[i] > bv)) { bv = v[i]; bi = i; }
    }
    int bid = bi < 0 ? 0x7FFFFFFF : lane + 32 * bi;
    // warp argmax: larger value wins, equal values -> lower id
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oid = __shfl_xor_sync(0xFFFFFFFFu, bid, off);
      const bool other_better = (oid != 0x7FFFFFFF) &&
                                (bid == 0x7FFFFFFF || ov > bv || (ov == bv && oid < bid));
      if (other_better) { bv = ov; bid = oid; }
    }
    if (j == 0) vmax = bv;
    if ((bid & 31) == lane) taken |= 1u << (bid >> 5);
    if (lane == j) { sel_v = bv; sel_id = bid; }
  }

  float w;
  const bool mine = lane < k;
  if (mode == 1) {  // top-k then softmax
    const float ex = mine ? expf(sel_v - vmax) : 0.0f;
    float s = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
    w = ex / s;
  } else {  // softmax over all E, then renormalise over the selected set
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
      if (lane + 32 * i < E) z += expf(v[i] - vmax);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, off);
    const float p = mine ? expf(sel_v - vmax) / z : 0.0f;
    float s = p;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
    w = p / s;
  }
  sel_id_out = sel_id;
  w_out = w;
}

template <int NPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                     int mode, int32_t* __restrict__ ids,
                                                     float* __restrict__ wts) {
  pdl_enter();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  if (t >= T) return;
  int sel_id;
  float w;
  route_token<NPL>(logits + size_t(t) * E, E, k, mode, lane, sel_id, w);
  if (lane < k) {
    ids[size_t(t) * k + lane] = sel_id;
    wts[size_t(t) * k + lane] = w;
  }
}

static cudaError_t launch_route(const float* logits, int T, int E, int k, int mode, int32_t* ids,
                                float* w, cudaStream_t s) {
  const int warps = 8;
  const dim3 grid((T + warps - 1) / warps), block(32 * warps);
  const int npl = (E + 31) / 32;
  ProfileScope prof(FT_KERNEL_ROUTE, s);
  auto kern = npl <= 1 ? route_kernel<1> : npl <= 2 ? route_kernel<2> : npl <= 4 ? route_kernel<4>
             : npl <= 8 ? route_kernel<8> : npl <= 16 ? route_kernel<16> : route_kernel<32>;
  return launch_pdl(kern, grid, block, 0, s, logits, T, E, k, mode, ids, w);
}

}  // namespace ftmoe
