// Combine: y[t, :] = sum_{j<k} w[t, j] * out_perm[pair_to_row[t*k + j], :],
// accumulated in fp32 in the order j = 0 .. k-1; out_perm and y are fp32.
//
// HBM-bound gather: each thread owns 4 consecutive hidden features (one
// 16-byte load per selected row), consecutive threads cover consecutive
// features of a token so every load and store is a fully used sector.
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace ftmoe {

__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ out_perm,
                                                      const int32_t* __restrict__ pair_to_row,
                                                      const float* __restrict__ w, int T, int k, int H,
                                                      int P, float4* __restrict__ y) {
  pdl_enter();
  const int vec_per_row = H / 4;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * vec_per_row) return;
  const int t = int(i / vec_per_row), c = int(i % vec_per_row);
  const int32_t* rows = pair_to_row + size_t(t) * k;
  const float* wt = w + size_t(t) * k;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  // eight selections at a time: their indices, weights and rows are all
  // requested before the first is used (one memory round trip per batch
  // instead of two per selection); the sum keeps the order j = 0 .. k-1
  for (int j0 = 0; j0 < k; j0 += 8) {
    int row[8];
    float wj[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      row[q] = j0 + q < k ? __ldg(rows + j0 + q) : -1;
      wj[q] = j0 + q < k ? __ldg(wt + j0 + q) : 0.0f;
    }
    float4 o[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const bool ok = row[q] >= 0 && row[q] < P;
      if (j0 + q < k && !ok) set_device_status(FT_DEV_BAD_INDEX);
      o[q] = ok ? __ldg(out_perm + size_t(row[q]) * vec_per_row + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (row[q] < 0 || row[q] >= P) continue;   // also the padding past k (row -1)
      acc.x = fmaf(wj[q], o[q].x, acc.x);
      acc.y = fmaf(wj[q], o[q].y, acc.y);
      acc.z = fmaf(wj[q], o[q].z, acc.z);
      acc.w = fmaf(wj[q], o[q].w, acc.w);
    }
  }
  y[size_t(t) * vec_per_row + c] = acc;
}

static cudaError_t launch_combine(const void* out_perm, const int32_t* pair_to_row, const float* w, int T,
                                  int k, int H, void* y, cudaStream_t s) {
  const long long n = (long long)T * (H / 4);
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  ProfileScope prof(FT_KERNEL_COMBINE, s);
  return launch_pdl(combine_kernel, dim3(unsigned(blocks)), dim3(threads), 0, s,
                    static_cast<const float4*>(out_perm), pair_to_row, w, T, k, H, T * k, static_cast<float4*>(y));
}

}  // namespace ftmoe
