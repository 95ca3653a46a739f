// ft_moe_permute_noalloc: the permutation of ft_moe_permute with its per-chunk
// expert counts kept in a fixed array of this module instead of a
// caller-supplied workspace.
//
// Who needs it: a caller that must not draw device memory at the moment of the
// call -- a host program with no device allocator of its own, or a runtime
// whose device memory is carved up once at start-up -- and so cannot hand
// ft_moe_permute the workspace it asks for when T*k > 1024.
//
// Scratch: kNoAllocScratchInts int32 (256 KiB) of file-scope device memory,
// enough for ceil(T*k / 1024) * E <= 65536 counts (for example T*k = 65536
// pairs over E = 1024 experts).  Larger inputs are rejected before anything is
// launched.  The histogram kernel writes every count that the scan and scatter
// kernels of the same call read, so the scratch needs no zeroing, at start-up
// or between calls.
//
// The device address of the scratch is looked up on every call that needs
// it, with the caller's device current (a host-side lookup, cheap next to the
// launches), so it stays right across devices and after a device reset.  The
// first call on a device may load this module's device code there: make it
// before any stream capture.  All calls on one device share the one scratch
// array, so two calls that may run at the same time (on two streams, or from
// two host threads) race on it: order them on one stream or with events.
#include "ftmoe.h"

namespace ftmoe {

constexpr int kNoAllocScratchInts = 65536;

static __device__ __align__(256) int32_t g_permute_scratch[kNoAllocScratchInts];

// Device address of g_permute_scratch on the current device.  In host code
// the array's name stands for the host-side shadow of the symbol, not a
// device address, so it is never passed to a kernel directly.
static cudaError_t permute_scratch(int32_t** out) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(out), g_permute_scratch);
}

}  // namespace ftmoe

extern "C" int ft_moe_permute_noalloc(const int32_t* ids, int T, int k, int E, int32_t* offsets,
                                      int32_t* perm_src, int32_t* pair_to_row, ft_stream_t stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || (long long)T * k > (1LL << 30))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_permute_noalloc: need 1 <= k <= E <= 1024");
  if (!offsets) return fail(FT_ERR_INVALID_ARG, "ft_moe_permute_noalloc: null pointer");
  if (T > 0 && (!ids || !perm_src || !pair_to_row))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_permute_noalloc: null pointer");
  const long long P = (long long)T * k;
  const long long nchunks = (P + kPermChunk - 1) / kPermChunk;
  if (nchunks > 1 && nchunks * E > kNoAllocScratchInts)
    return fail(FT_ERR_INVALID_ARG,
                "ft_moe_permute_noalloc: ceil(T*k/1024)*E exceeds the 65536-count scratch; "
                "use ft_moe_permute with a workspace");
  const cudaStream_t s = S(stream);
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(offsets, 0, size_t(E + 1) * sizeof(int32_t), s);
    return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_permute_noalloc");
  }
  int32_t* counts = nullptr;
  if (nchunks > 1) {
    const cudaError_t e = permute_scratch(&counts);
    if (e != cudaSuccess) return cuda_fail(e, "ft_moe_permute_noalloc: scratch address");
  }
  // the launches of ft_moe_permute, with the scratch in place of the workspace
  const cudaError_t e = launch_permute(ids, T, k, E, offsets, perm_src, pair_to_row, counts, s);
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_permute_noalloc");
}
