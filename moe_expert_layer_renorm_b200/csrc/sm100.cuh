// Thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers (with bounded waits), TMA tensor loads, cp.async, and the
// tcgen05 family (TMEM alloc, tcgen05.st/ld, tcgen05.mma kind::f16, commit).
//
// Every wait in this library is bounded: a wait that exceeds the limit
// records an error code in the library's device status word and returns
// false, so a kernel never spins forever.
#pragma once
#include <utility>
#include <cstdint>
#include <cuda_runtime.h>

namespace ftmoe {

// Device status word (error codes are FT_DEV_* below).  The library is built
// as one translation unit, so this header is included exactly once.
__device__ int g_device_status = 0;
// Detail of the first recorded status: {code, block, warp, tag, counter, unit, elapsed_us, 0}.
__device__ long long g_device_status_detail[8];

enum : int {
  FT_DEV_OK = 0,
  FT_DEV_WAIT_TIMEOUT = 1,
  FT_DEV_NOT_RESIDENT = 2,   // a non-empty expert group maps to slot -1
  FT_DEV_BAD_INDEX = 3,      // an id or slot index outside its range
  FT_DEV_F16_RANGE = 4,      // an intermediate exceeded the f16 range and was saturated
};

__device__ __forceinline__ void set_device_status(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// Record `code` with where it happened; only the first caller's detail is kept.
__device__ __forceinline__ void set_device_status_detail(int code, int tag, long long counter, long long unit,
                                                         long long elapsed_us) {
  if (atomicCAS(&g_device_status, 0, code) == 0) {
    g_device_status_detail[0] = code;
    g_device_status_detail[1] = blockIdx.x;
    g_device_status_detail[2] = threadIdx.x >> 5;
    g_device_status_detail[3] = tag;
    g_device_status_detail[4] = counter;
    g_device_status_detail[5] = unit;
    g_device_status_detail[6] = elapsed_us;
    __threadfence();
  }
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------ mbarrier ---

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}"
               ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n}"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
               " selp.b32 %0, 1, 0, p;\n}"
               : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed.  Gives up after
// ~1 s of wall time, records FT_DEV_WAIT_TIMEOUT and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++n & 255u) == 0 && globaltimer_ns() - t0 > 1000000000ull) {
      set_device_status(FT_DEV_WAIT_TIMEOUT);
      return false;
    }
  }
}

// ----------------------------------------------------------------- TMA ---

// 3-D tiled TMA load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// 4-D tiled TMA load (no multicast).
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y, int z,
                                            int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

// One weight box (codes: 128 B of each row; scales: 16 B) of 256-K stage ws,
// rows from y, slot `slot`.  Row-major slots use 3-D maps whose x is the
// byte column (stage ws starts at ws * stage_bytes); stage-tiled slots use
// 4-D maps with the stage as a dimension of its own (x = 0).
__device__ __forceinline__ void tma_load_weights(void* smem_dst, const void* tmap, uint64_t* bar, int tiled,
                                                 int stage_bytes, int ws, int y, int slot) {
  if (tiled)
    tma_load_4d(smem_dst, tmap, bar, 0, y, ws, slot);
  else
    tma_load_3d(smem_dst, tmap, bar, ws * stage_bytes, y, slot);
}

// 2-D tiled TMA load (no multicast).
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// TMA row gather (no multicast): four rows y0..y3 of a 2-D tensor whose map
// has a one-row box, columns [x, x + box width), written as four consecutive
// rows of the destination tile.
__device__ __forceinline__ void tma_gather4(void* smem_dst, const void* tmap, uint64_t* bar, int x, int y0,
                                            int y1, int y2, int y3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3)
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

// ------------------------------------------------------------ cp.async ---

// 16-byte async copy global -> shared; src_bytes = 0 zero-fills the chunk.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
               ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------- TMEM ---

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_result)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Each thread of the warp writes 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
        "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
        "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
        "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr) : "memory");
}

// ------------------------------------------------------------- tcgen05 ---

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulate, A and B
// both bf16 (ab_f16 = false) or both f16, both K-major, shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_f16(int M, int N, bool ab_f16 = false) {
  return (1u << 4)                                     // D format: f32
       | ((ab_f16 ? 0u : 1u) << 7)                     // A format: bf16 (1) / f16 (0)
       | ((ab_f16 ? 0u : 1u) << 10)                    // B format
       | (0u << 15) | (0u << 16)                       // A, B K-major
       | (uint32_t(N >> 3) << 17)
       | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major operand stored in the
// 128-byte swizzled layout: rows of 128 B, 8-row atoms of 1024 B.
__device__ __forceinline__ uint64_t make_sdesc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFFu);          // start address
  d |= uint64_t(1u) << 16;                              // leading byte offset (unused for SW128 K-major)
  d |= uint64_t(1024u >> 4) << 32;                      // stride byte offset: 8 rows x 128 B
  d |= uint64_t(1u) << 46;                              // descriptor version (sm_100)
  d |= uint64_t(2u) << 61;                              // layout: 128-byte swizzle
  return d;
}

// D[tmem_d] (+)= A[tmem_a] * B[smem desc]^T, one CTA, kind::f16.
__device__ __forceinline__ void mma_ts_f16(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}"
      ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// D[tmem_d] (+)= A[smem desc] * B[smem desc]^T, one CTA, kind::f16.
__device__ __forceinline__ void mma_ss_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// The same, always accumulating (no predicate to set up between MMAs).
__device__ __forceinline__ void mma_ts_f16_acc(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc) {
  asm volatile("tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, 1;"
               ::"r"(tmem_d), "r"(tmem_a), "l"(bdesc), "r"(idesc) : "memory");
}

// Arrive on `bar` once all tcgen05.mma previously issued by this thread finish.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// Named barrier for a subset of warps.
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Programmatic dependent launch.  Every hot-path kernel starts with this:
// wait until the grids it depends on have completed and their memory is
// visible (a no-op when it was launched without such a dependency), then let
// the next grid in the stream begin launching, so that its set-up overlaps
// this grid's work instead of following it.
__device__ __forceinline__ void pdl_enter() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// The two halves separately: a kernel that fills whole SMs triggers its
// dependents only as its CTAs finish, so that their early CTAs do not take
// SM resources from it while it runs.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Launch with the programmatic-stream-serialisation attribute: the kernel
// may start before the previous kernel in the stream ends, and waits for it
// in pdl_enter().  Captured into CUDA graphs as a programmatic edge.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace ftmoe
