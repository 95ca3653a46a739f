// Self-test of the kernels' bounded waits (ft_selftest_wait_timeout): one CTA
// of two warps, each waiting on an mbarrier whose phase nothing completes,
// through the same Abort::wait the expert GEMMs use.  Warp 0's wait runs out
// after ~1 s of wall time, records FT_DEV_WAIT_TIMEOUT with its detail and
// raises the CTA's abort flag; warp 1, polling the flag inside its own wait,
// then leaves too, before its own limit (it starts 0.5 s later).  Both
// report whether their wait gave up.  The kernel ends normally, so the
// context stays usable: this is how the failure path is exercised without a
// fault.
#include "sm100.cuh"

namespace ftmoe {

__global__ void __launch_bounds__(64) wait_selftest_kernel(int32_t* out) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  const Abort ab{&abort_flag};
  bool ok;
  if (warp == 0) {
    ok = ab.wait(&bar[0], 0, kTagBFull, /*counter=*/7, /*unit=*/3);
  } else {
    // start 0.5 s later, so that warp 0's limit is the one that runs out
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 500000000ull) {
    }
    ok = ab.wait(&bar[1], 0, kTagWFull, 0, 0);
  }
  if ((threadIdx.x & 31) == 0) out[warp] = ok ? 0 : 1;
}

static cudaError_t launch_wait_selftest(int32_t* out, cudaStream_t s) {
  wait_selftest_kernel<<<1, 64, 0, s>>>(out);
  return cudaGetLastError();
}

}  // namespace ftmoe
