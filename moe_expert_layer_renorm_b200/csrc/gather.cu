// Row gather: dst[i, :] = src[idx[i] / div, :] for i in [0, n), rows of a
// fixed byte length (a multiple of 16).  The expert-parallel exchange uses it
// twice: a sender lays out the activation row of each routed pair in
// expert order (idx = perm_src, div = k), so that each destination rank's
// rows are contiguous; a receiver puts its expert outputs back in the order
// the rows arrived in (div = 1) before returning them.
//
// A plain HBM copy: one 16-byte vector per thread and iteration, consecutive
// threads on consecutive vectors of a row, a grid of a few CTAs per SM
// striding over the rows.  An index outside [0, n_src) sets
// FT_DEV_BAD_INDEX and writes a zero row.
#include "sm100.cuh"

namespace ftmoe {

__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ src, int n_src,
                                                          const int32_t* __restrict__ idx, int div, int n,
                                                          int vec_per_row, uint4* __restrict__ dst) {
  pdl_enter();
  const long long total = (long long)n * vec_per_row;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int r = int(i / vec_per_row), c = int(i % vec_per_row);
    const int v = __ldg(idx + r);
    const int s = v >= 0 ? v / div : -1;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (s >= 0 && s < n_src)
      val = __ldg(src + size_t(s) * vec_per_row + c);
    else if (c == 0)
      set_device_status(FT_DEV_BAD_INDEX);
    dst[i] = val;
  }
}

static cudaError_t launch_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx, int div,
                                      int n, void* dst, int num_sms, cudaStream_t s) {
  const int vec_per_row = row_bytes / 16;
  const long long total = (long long)n * vec_per_row;
  const int threads = 256;
  const long long want = (total + threads - 1) / threads;
  const int blocks = int(std::min<long long>(want, (long long)num_sms * 8));
  ProfileScope prof(FT_KERNEL_GATHER, s);
  return launch_pdl(gather_rows_kernel, dim3(unsigned(blocks)), dim3(threads), 0, s,
                    static_cast<const uint4*>(src), n_src, idx, div, n, vec_per_row, static_cast<uint4*>(dst));
}

}  // namespace ftmoe
