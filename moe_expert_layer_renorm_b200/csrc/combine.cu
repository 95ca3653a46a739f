// Combine: y[t, :] = bf16( sum_{j<k} w[t, j] * out_perm[pair_to_row[t*k + j], :] ),
// accumulated in fp32 in the order j = 0 .. k-1.
//
// HBM-bound gather: each thread owns 8 consecutive hidden features (one
// 16-byte load per selected row), consecutive threads cover consecutive
// features of a token so every load and store is a fully used sector.
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace ftmoe {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ out_perm,
                                                      const int32_t* __restrict__ pair_to_row,
                                                      const float* __restrict__ w, int T, int k, int H,
                                                      int P, uint4* __restrict__ y) {
  const int vec_per_row = H / 8;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * vec_per_row) return;
  const int t = int(i / vec_per_row), c = int(i % vec_per_row);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int j = 0; j < k; ++j) {
    const int row = __ldg(pair_to_row + size_t(t) * k + j);
    if (row < 0 || row >= P) { set_device_status(FT_DEV_BAD_INDEX); continue; }
    const float wj = __ldg(w + size_t(t) * k + j);
    float f[8];
    bf16x8_to_f32(__ldg(out_perm + size_t(row) * vec_per_row + c), f);
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = fmaf(wj, f[q], acc[q]);
  }
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  y[size_t(t) * vec_per_row + c] = o;
}

static cudaError_t launch_combine(const void* out_perm, const int32_t* pair_to_row, const float* w, int T,
                                  int k, int H, void* y, cudaStream_t s) {
  const long long n = (long long)T * (H / 8);
  const int threads = 256;
  const long long blocks = (n + threads - 1) / threads;
  ProfileScope prof(FT_KERNEL_COMBINE, s);
  combine_kernel<<<dim3(unsigned(blocks)), threads, 0, s>>>(static_cast<const uint4*>(out_perm), pair_to_row, w,
                                                            T, k, H, T * k, static_cast<uint4*>(y));
  return cudaGetLastError();
}

}  // namespace ftmoe
