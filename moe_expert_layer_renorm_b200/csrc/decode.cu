// Expert FFN, decode variant: both grouped GEMMs of the layer (gate/up with
// SwiGLU, then down) in ONE persistent launch, for groups of at most 16 token
// rows.  Bound by the NVFP4 weight bytes read from HBM.
//
// Why not tcgen05 here: with a handful of token rows per expert the MMA is a
// tall-skinny product, and every tcgen05.mma instruction consumes at most
// 128 (M side) x 16 (K) weights per ~100 cycles of its SM when the weights are
// the M operand; as the N operand the dequantised tile must make a round trip
// through shared memory.  Streaming at HBM rate needs ~35-50 weights per clock
// per SM, so the weights flow from TMA-staged shared memory through registers
// straight into warp-level MMA fragments (mma.sync m16n8k16, f16 x f16 ->
// fp32): 256 weights per instruction, and the tensor cores do the FMAs.
//
// Work units (built on the device by ffn_prep_kernel), in one queue:
//   gate/up unit: 128 features (their 128 gate rows and 128 up rows) of one
//                 expert x one group of <= 16 token rows x a K range;
//   down unit:    256 rows of the down matrix x the same token group x a K range.
// CTAs take units from a global counter in queue order (all gate/up units
// first), so a long unit never waits behind a short one and no SM idles at a
// wave boundary.  A down unit reads h rows written by the gate/up units of
// its token group: its token loader waits (bounded) until those have all
// published; every unit it waits on was taken earlier by a running CTA, so
// the wait always ends.  The down unit's weights stream in meanwhile.
//
// CTA (19 warps):
//   warps 0-15  compute: warp w owns 16 rows of the 256-row tile (gate/up:
//               the gate and up rows of features 8w .. 8w+7) and all of each
//               256-K stage, so it finishes its outputs alone: no partial
//               sums change hands inside the CTA and the epilogue needs no
//               barrier.
//   warp 16     takes units from the queue; TMA of the 256 weight rows (two
//               128-row boxes of codes, 128-byte swizzle, and of scales)
//   warp 17     TMA of the unit's token rows (16-row boxes of the permuted f16
//               activations or of h), after the dependency wait for down units
//   warp 18     publishes each gate/up unit's finished h rows to other CTAs
//               with one release, so compute warps never wait on a fence
//
// K permutation.  A dot product may visit K in any order as long as both
// operands use the same order.  For MMA step i (0..7) of a 128-K half stage,
// thread t of each quad supplies logical k in {2t, 2t+1, 2t+8, 2t+9}; they
// are mapped to physical k = 32 t + 4 i + {0, 1, 2, 3}.  So a thread's codes
// for all eight steps are 32 consecutive K of its row (one 16-byte load, two
// scale bytes), and its token values are 32 consecutive K of the token row
// (four 16-byte loads per token tile).
#include <cuda.h>
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

constexpr int kDecThreads = 19 * 32;
constexpr int kDecRows = 256;      // weight rows per CTA tile (down); gate/up: 128 features x 2
constexpr int kDecFeat1 = 128;     // gate/up features per tile
constexpr int kDecBN = 16;         // token rows per unit
constexpr int kDecStageK = 256;
constexpr int kDecStages = 4;
constexpr int kDecUnitRing = 2;    // units a CTA holds: the one in compute and the next
constexpr int kDecCodes = kDecRows * 128;                 // 256 rows x 128 B of codes
constexpr int kDecWStageBytes = kDecCodes + kDecRows * 16; // + 256 rows x 16 B of scales
constexpr int kDecBBoxBytes = kDecBN * 128;               // 64 K x 16 rows of f16
constexpr int kDecBStageBytes = 4 * kDecBBoxBytes;        // 256 K
constexpr int kDecStageBytes = kDecWStageBytes + kDecBStageBytes;
constexpr int kDecSmemBytes =
    1024 + kDecStages * kDecStageBytes + (2 * kDecStages + 2 * kDecUnitRing + 2) * 8 + 128;
constexpr int kDecPartialBytes = 16 * 2 * 32 * 16;        // one unit's split-K partial sums (warp x n-tile x lane)
static_assert(kDecStageBytes % 1024 == 0, "stage alignment");
static_assert(kDecSmemBytes <= 227 * 1024, "shared memory budget");

// Barrier tag of the down unit's wait for its h rows.
constexpr int kTagDep = 9;

struct DecodeParams {
  FfnParams g[2];      // [0] gate/up + SwiGLU (h out), [1] down (out_perm out)
  int* queue;          // next queue position to take (zeroed by ffn_prep_kernel)
  int* tile_done;      // per token tile: gate/up epilogue warps (16 per m-tile) that published h
  int mt1;             // gate/up m-tiles (128 features) per token tile
  int mt2;             // down m-tiles (256 rows) per token tile
};

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int atom_acq_rel_gpu_add(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One queue entry, decoded.
struct DecUnit {
  int gemm;            // 0 gate/up, 1 down
  int u;               // index within its GEMM's unit list
  int e, slot;         // expert and its slot in the pool
  int mt, rb, nr;      // m-tile, first permuted row, rows (<= 16)
  int split, ws0, ws1; // split index, K-stage range
  int tile;            // token tile (same tiling for both GEMMs)
};

// Queue position q is unit q of gate/up (q < n1) or unit q - n1 of down.
__device__ __forceinline__ int4 unit_desc(const DecodeParams& p, int q, int n1) {
  return q < n1 ? p.g[0].units[q] : p.g[1].units[q - n1];
}

// v: the unit's descriptor {expert | slot << 10, m-tile, first row, rows | split << 16}
__device__ __forceinline__ DecUnit decode_unit(const DecodeParams& p, int q, int n1, const int4 v) {
  DecUnit d;
  d.gemm = q < n1 ? 0 : 1;
  d.u = d.gemm ? q - n1 : q;
  const FfnParams& g = p.g[d.gemm];
  d.e = v.x & 1023; d.slot = v.x >> 10;
  d.mt = v.y; d.rb = v.z; d.nr = v.w & 0xFFFF;
  d.split = v.w >> 16;
  d.ws0 = d.split * g.stages_per_split;
  d.ws1 = min(g.nkw, d.ws0 + g.stages_per_split);
  const int per_tile = (d.gemm ? p.mt2 : p.mt1) * g.splits;
  d.tile = d.u / per_tile;
  return d;
}

// Rows of the 256-row stage that warp w covers as the A rows g and g + 8 of
// its m16 tiles.  Gate/up stages hold the 128 gate rows then the 128 up rows
// of the same features; warp w takes features 8w .. 8w+7 -- their gate rows
// as A rows g and their up rows as A rows g + 8 -- so each thread ends up
// with both halves of its SwiGLUs.  Down stages: rows 16w .. 16w+15.
//
// Inside each group of 8 rows, A row g is row dec_sub(g) = g/2 + 4 (g % 2):
// the two quads that share a 16-byte load's 8-lane phase (g = 2j, 2j + 1)
// then read rows whose 128-byte swizzle phases differ in bit 2, so their
// eight 16-byte code chunks fall in eight different bank groups (with rows
// g and g + 1 both quads' chunks landed in the same four).  The outputs
// follow the same map.
__device__ __forceinline__ int dec_sub(int g) { return (g >> 1) | ((g & 1) << 2); }
__device__ __forceinline__ int dec_row_lo(int gemm, int w, int g) {
  return gemm ? 16 * w + dec_sub(g) : 8 * w + dec_sub(g);
}
__device__ __forceinline__ int dec_row_hi(int gemm, int w, int g) {
  return gemm ? 16 * w + 8 + dec_sub(g) : kDecFeat1 + 8 * w + dec_sub(g);
}

// One 256-K stage for this warp: its 16 rows x 256 K x NT token tiles of 8.
template <int NT, int FMT>
__device__ __forceinline__ void dec_stage(const uint8_t* st, int r_lo, int r_hi, int g, int t, int blo, int bhi,
                                          float (&acc)[NT][4]) {
  const uint8_t* bst = st + kDecWStageBytes;
#pragma unroll
  for (int h = 0; h < 2; ++h) {   // 128-K halves: thread t covers K 128h + 32t .. +31
    const uint8_t* bbox = bst + (2 * h + (t >> 1)) * kDecBBoxBytes;
    const int chunk = 4 * h + t;   // 16-byte chunk of the 128-byte codes row: 32 codes
    const uint4 clo = *reinterpret_cast<const uint4*>(st + r_lo * 128 + ((chunk ^ (r_lo & 7)) << 4));
    const uint4 chi = *reinterpret_cast<const uint4*>(st + r_hi * 128 + ((chunk ^ (r_hi & 7)) << 4));
    const uint32_t slo = *reinterpret_cast<const uint16_t*>(st + kDecCodes + r_lo * 16 + 8 * h + 2 * t);
    const uint32_t shi = *reinterpret_cast<const uint16_t*>(st + kDecCodes + r_hi * 16 + 8 * h + 2 * t);
    const uint32_t wlo[4] = {clo.x, clo.y, clo.z, clo.w};
    const uint32_t whi[4] = {chi.x, chi.y, chi.z, chi.w};
    // the thread's 32 K span two 16-K scale blocks: words 0, 1 and words 2, 3
    uint32_t sl2[2], sh2[2];
    if (FMT == FT_SCALE_NVFP4) {   // both blocks' scales in one conversion, each then broadcast to a pair
      e4m3x2_to_pairs(slo, sl2[0], sl2[1]);
      e4m3x2_to_pairs(shi, sh2[0], sh2[1]);
    } else {
      sl2[0] = scale_pair_to_f16x2<FMT>(slo & 0xFFu, blo); sl2[1] = scale_pair_to_f16x2<FMT>(slo >> 8, blo);
      sh2[0] = scale_pair_to_f16x2<FMT>(shi & 0xFFu, bhi); sh2[1] = scale_pair_to_f16x2<FMT>(shi >> 8, bhi);
    }
#pragma unroll
    for (int wd = 0; wd < 4; ++wd) {   // word wd: 8 K = two MMA steps
      const int cb = (t & 1) * 4 + wd;   // the token values of those 8 K: 16-byte chunk of the box row
      uint4 bv[NT];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int row = 8 * n + g;
        bv[n] = *reinterpret_cast<const uint4*>(bbox + row * 128 + ((cb ^ (row & 7)) << 4));
      }
      const uint32_t sl = sl2[wd >> 1], sh = sh2[wd >> 1];
      uint32_t qlo[4], qhi[4];
      e2m1x8_to_f16x2(wlo[wd], qlo);
      e2m1x8_to_f16x2(whi[wd], qhi);
#pragma unroll
      for (int p = 0; p < 2; ++p) {   // physical k 4p + {0,1} (a0/a1, b0) and + {2,3} (a2/a3, b1)
        const uint32_t a0 = hmul2_f16(qlo[2 * p], sl), a1 = hmul2_f16(qhi[2 * p], sh);
        const uint32_t a2 = hmul2_f16(qlo[2 * p + 1], sl), a3 = hmul2_f16(qhi[2 * p + 1], sh);
#pragma unroll
        for (int n = 0; n < NT; ++n)
          mma_f16_16816(acc[n], a0, a1, a2, a3, p ? bv[n].z : bv[n].x, p ? bv[n].w : bv[n].y);
      }
    }
  }
}

// Per-unit epilogue constants, loaded by the weight producer while the unit
// streams in, and handed over through the unit ring.
struct DecConsts {
  float g0, g1;        // global scales: gate and up (gate/up unit) or down twice
};

__device__ __forceinline__ DecConsts dec_consts(const DecodeParams& p, const DecUnit& d) {
  const FfnParams& G = p.g[d.gemm];
  const uint8_t* sbase = G.pool + size_t(d.slot) * size_t(G.slot_bytes);
  DecConsts c;
  c.g0 = __ldg(reinterpret_cast<const float*>(sbase + G.global_off[0]));
  c.g1 = __ldg(reinterpret_cast<const float*>(sbase + G.global_off[1]));
  return c;
}

// Epilogue of warp w for its 16 rows.  With split-K across CTAs the warp
// first leaves its partial sums; the last split to arrive adds all splits
// in a fixed order and finishes.  Returns true if this warp stored the
// outputs.
template <int NT>
__device__ __forceinline__ bool dec_epilogue(const DecodeParams& p, const DecUnit& d, const DecConsts& c, int w,
                                             int lane, float (&acc)[NT][4], const float (&ts)[NT][2]) {
  const FfnParams& G = p.g[d.gemm];
  const int g = lane >> 2, t = lane & 3;
  if (G.splits > 1) {
    float4* part = reinterpret_cast<float4*>(G.partials);
    constexpr int kPer = kDecPartialBytes / 16;
    const int slot = (w * 2) * 32 + lane;
#pragma unroll
    for (int n = 0; n < NT; ++n)
      part[size_t(d.u) * kPer + slot + n * 32] = make_float4(acc[n][0], acc[n][1], acc[n][2], acc[n][3]);
    __syncwarp();
    int last = 0;
    if (lane == 0) last = atom_acq_rel_gpu_add(G.counters + (d.u / G.splits) * 16 + w, 1) == G.splits - 1;
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return false;
    if (lane == 0) G.counters[(d.u / G.splits) * 16 + w] = 0;   // every split has arrived: ready for the next call
    const int u0 = d.u - d.split;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < G.splits; ++sp) {   // fixed order: the same sums whoever arrives last
        const float4 v = __ldcg(part + size_t(u0 + sp) * kPer + slot + n * 32);
        s.x += v.x; s.y += v.y; s.z += v.z; s.w += v.w;
      }
      acc[n][0] = s.x; acc[n][1] = s.y; acc[n][2] = s.z; acc[n][3] = s.w;
    }
  }
  if (d.gemm == 0) {
    const int f = d.mt * kDecFeat1 + 8 * w + dec_sub(g);   // the feature of rows r_lo (gate) and r_hi (up)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 8 * n + 2 * t + e;
        if (r < d.nr && f < G.M) {
          store_out<2>(G.out, size_t(d.rb + r) * G.M + f,
                       silu_mul(c.g0 * kRowNormInv * acc[n][e], c.g1 * kRowNormInv * acc[n][2 + e], ts[n][e]));
        }
      }
  } else {
    const int f = d.mt * kDecRows + 16 * w + dec_sub(g);   // row r_lo; r_hi is f + 8
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 8 * n + 2 * t + e;
        if (r < d.nr) {
          float* o = static_cast<float*>(G.out) + size_t(d.rb + r) * G.M;
          if (f < G.M) o[f] = down_out(c.g0, acc[n][e], ts[n][e]);
          if (f + 8 < G.M) o[f + 8] = down_out(c.g0, acc[n][2 + e], ts[n][e]);
        }
      }
  }
  return true;
}

// Barrier tag of the unit ring.
constexpr int kTagUnit = 10;

// Main loop and epilogue of one unit for compute warp w.  `si` counts stages
// consumed by this CTA.  The unit's ring slot is released after the main
// loop, so a CTA takes a new unit from the queue only when it has finished
// computing the one before the current one: no CTA hoards small units while
// others idle.  Returns false if a wait gave up (the kernel then winds down).
template <int NT, int FMT>
__device__ bool dec_unit(const DecodeParams& p, const DecUnit& d, uint8_t* smem, uint64_t* full, uint64_t* empty,
                         const Abort& ab, uint64_t* unit_free, const int4* unit_ent, uint64_t* hpub, int* hcount,
                         int gu, uint32_t& si, int q, int w, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const int r_lo = dec_row_lo(d.gemm, w, g), r_hi = dec_row_hi(d.gemm, w, g);
  // MXFP4: the power of two each matrix's global takes out of its scales
  // (gate/up: gate rows lo, up rows hi; down: both)
  int blo = 0, bhi = 0;
  if (FMT == FT_SCALE_MXFP4) {
    const FfnParams& G = p.g[d.gemm];
    const uint8_t* sbase = G.pool + size_t(d.slot) * size_t(G.slot_bytes);
    blo = mx_bias(__ldg(reinterpret_cast<const float*>(sbase + G.global_off[0])));
    bhi = mx_bias(__ldg(reinterpret_cast<const float*>(sbase + G.global_off[1])));
  }
  // the token rows' factors f_r (see silu_mul), loaded now, used in the epilogue
  float ts[NT][2];
  const float* rs = p.g[d.gemm].rowscale;
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 8 * n + 2 * t + e;
      ts[n][e] = rs != nullptr && r < d.nr ? __ldg(rs + d.rb + r) : 1.0f;
    }
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.0f;

  for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
    const int s = si % kDecStages;
    if (!__all_sync(0xFFFFFFFFu, ab.wait(&full[s], (si / kDecStages) & 1, kTagWFull, si, q))) return false;
    dec_stage<NT, FMT>(smem + s * kDecStageBytes, r_lo, r_hi, g, t, blo, bhi, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }
  DecConsts c;   // written by the weight producer before the last stage (acquired above)
  {
    const int4 ce = *unit_ent;
    c.g0 = __int_as_float(ce.y); c.g1 = __int_as_float(ce.z);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(unit_free);   // the queue may hand this CTA its next-but-one unit
  const bool fin = dec_epilogue<NT>(p, d, c, w, lane, acc, ts);
  if (d.gemm == 0) {   // gate/up: hand the h rows to the publisher
    __syncwarp();
    if (fin && lane == 0) atomicAdd(&hcount[gu & 1], 1);
    mbar_arrive(&hpub[gu & 1]);   // after this thread's stores (release)
  }
  return true;
}

// Bounded wait of a down unit's token loader for the h rows of its token
// tile: all gate/up m-tiles of the tile published (each of the 16 compute
// warps publishes its quarter of its row group).
__device__ bool dec_wait_h(const DecodeParams& p, const DecUnit& d, const Abort& ab, int q) {
  const int* flag = p.tile_done + d.tile;
  const int target = 16 * p.mt1;
  if (ld_acquire_gpu(flag) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (ld_acquire_gpu(flag) < target) {
    __nanosleep(128);
    if ((++n & 15u) == 0) {
      if (*ab.flag) return false;
      const uint64_t dt = globaltimer_ns() - t0;
      if (dt > 1000000000ull) {
        set_device_status_detail(FT_DEV_WAIT_TIMEOUT, kTagDep, d.tile, q, (long long)(dt / 1000));
        *ab.flag = 1;
        return false;
      }
    }
  }
  return true;
}

// Wait (bounded) for the last stages a producer issued, so that no TMA write
// into this CTA's shared memory is in flight when it exits.
__device__ void dec_drain(uint64_t* full, uint32_t si) {
  for (uint32_t k = (si > kDecStages ? si - kDecStages : 0); k < si; ++k) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&full[k % kDecStages], (k / kDecStages) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
  }
}

template <int FMT>
__global__ void __launch_bounds__(kDecThreads, 1)
ffn_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_c0,
                  const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_c1,
                  const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_c2,
                  const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_h) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDecStages * kDecStageBytes);
  uint64_t* empty = full + kDecStages;
  uint64_t* ufull = empty + kDecStages;
  uint64_t* uempty = ufull + kDecUnitRing;
  uint64_t* hpub = uempty + kDecUnitRing;   // [2] by gate/up ordinal parity: all compute threads stored h
  // ring entries: {queue position, then (before the unit's last stage lands)
  // the epilogue constants: global scale bits x2}
  int4* uent = reinterpret_cast<int4*>(hpub + 2);
  int4* udesc = uent + kDecUnitRing;   // [kDecUnitRing] the unit's descriptor, read once by the producer
  int* hcount = reinterpret_cast<int*>(udesc + kDecUnitRing);   // [2] warps that finished their h rows
  int* abort_flag = hcount + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecStages; ++i) { mbar_init(&full[i], 2); mbar_init(&empty[i], 16); }
    for (int i = 0; i < kDecUnitRing; ++i) { mbar_init(&ufull[i], 1); mbar_init(&uempty[i], 18); }
    for (int i = 0; i < 2; ++i) { mbar_init(&hpub[i], 512); hcount[i] = 0; }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 16 && lane == 0) {
    prefetch_tmap(&tm_c0); prefetch_tmap(&tm_s0); prefetch_tmap(&tm_c1);
    prefetch_tmap(&tm_s1); prefetch_tmap(&tm_c2); prefetch_tmap(&tm_s2);
  }
  if (warp == 17 && lane == 0) { prefetch_tmap(&tm_x); prefetch_tmap(&tm_h); }
  __syncthreads();
  const Abort ab{abort_flag};
  const int n1 = *p.g[0].num_units;
  const int ntot = n1 + *p.g[1].num_units;

  if (warp == 16) {
    // ------------------------------------------- queue + weight TMA ---
    if (lane == 0) {
      uint32_t si = 0;
      bool ok = true;
      // The next unit is taken from the queue (and its descriptor fetched)
      // while the current one's stages are issued, so that the global
      // round trips do not open a gap in the weight stream; it is handed to
      // the consumers only once the ring has room for it.
      int next_q = atomicAdd(p.queue, 1);
      int4 next_raw = next_q < ntot ? unit_desc(p, next_q, n1) : make_int4(0, 0, 0, 0);
      for (int j = 0; ok; ++j) {
        const int us = j % kDecUnitRing;
        if (!(ok = ab.wait(&uempty[us], ((j / kDecUnitRing) & 1) ^ 1, kTagUnit, j, -3))) break;
        const int q = next_q < ntot ? next_q : -1;
        const int4 raw = next_raw;
        if (q >= 0) next_q = atomicAdd(p.queue, 1);   // used after this unit's stages are issued
        udesc[us] = raw;
        uent[us].x = q;
        mbar_arrive(&ufull[us]);
        if (q < 0) break;
        const DecUnit d = decode_unit(p, q, n1, raw);
        const DecConsts c = dec_consts(p, d);
        const int slot = d.slot;
        const CUtensorMap* c0 = d.gemm ? &tm_c2 : &tm_c0;
        const CUtensorMap* c1 = d.gemm ? &tm_c2 : &tm_c1;
        const CUtensorMap* s0 = d.gemm ? &tm_s2 : &tm_s0;
        const CUtensorMap* s1 = d.gemm ? &tm_s2 : &tm_s1;
        const int y0 = d.gemm ? d.mt * kDecRows : d.mt * kDecFeat1;
        const int y1 = d.gemm ? y0 + 128 : y0;
        for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
          const int s = si % kDecStages;
          if (!(ok = ab.wait(&empty[s], ((si / kDecStages) & 1) ^ 1, kTagWEmpty, si, q))) break;
          if (ws == d.ws1 - 1)   // published by this stage's arrival (release) to the compute warps
            uent[us] = make_int4(q, __float_as_int(c.g0), __float_as_int(c.g1), 0);
          mbar_arrive_expect_tx(&full[s], kDecWStageBytes);
          uint8_t* st = smem + s * kDecStageBytes;
          const int tl = p.g[0].tiled;
          tma_load_weights(st, c0, &full[s], tl, 128, ws, y0, slot);
          tma_load_weights(st + 128 * 128, c1, &full[s], tl, 128, ws, y1, slot);
          tma_load_weights(st + kDecCodes, s0, &full[s], tl, 16, ws, y0, slot);
          tma_load_weights(st + kDecCodes + 128 * 16, s1, &full[s], tl, 16, ws, y1, slot);
        }
        next_raw = next_q < ntot ? unit_desc(p, next_q, n1) : make_int4(0, 0, 0, 0);
      }
      dec_drain(full, si);
    }
  } else if (warp == 17) {
    // ------------------------------------------------- token TMA ---
    if (lane == 0) {
      uint32_t si = 0;
      bool ok = true;
      for (int j = 0; ok; ++j) {
        const int us = j % kDecUnitRing;
        if (!(ok = ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -1))) break;
        const int q = uent[us].x;
        if (q < 0) { mbar_arrive(&uempty[us]); break; }
        const DecUnit d = decode_unit(p, q, n1, udesc[us]);
        if (d.gemm == 1) {
          if (!(ok = dec_wait_h(p, d, ab, q))) break;
          fence_proxy_async_global();   // the h rows were written by generic stores
        }
        const CUtensorMap* act = d.gemm ? &tm_h : &tm_x;
        for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
          const int s = si % kDecStages;
          if (!(ok = ab.wait(&empty[s], ((si / kDecStages) & 1) ^ 1, kTagBEmpty, si, q))) break;
          mbar_arrive_expect_tx(&full[s], kDecBStageBytes);
          uint8_t* bst = smem + s * kDecStageBytes + kDecWStageBytes;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_2d(bst + bx * kDecBBoxBytes, act, &full[s], ws * kDecStageK + bx * 64, d.rb);
        }
        mbar_arrive(&uempty[us]);
      }
      dec_drain(full, si);
    }
  } else if (warp == 18) {
    // --------------------------------------------------- publisher ---
    // For each gate/up unit: once all compute threads stored their h rows,
    // add the number of warps that finished to the token tile's count with
    // one release (down units' token loaders acquire it).  The ring slot is
    // released only after publishing, which bounds how far the compute
    // warps run ahead of this warp.
    if (lane == 0) {
      int ngu = 0;
      for (int j = 0;; ++j) {
        const int us = j % kDecUnitRing;
        if (!ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -4)) break;
        const int q = uent[us].x;
        if (q < 0) { mbar_arrive(&uempty[us]); break; }
        const DecUnit d = decode_unit(p, q, n1, udesc[us]);
        if (d.gemm == 0) {
          const int hb = ngu & 1;
          if (!ab.wait(&hpub[hb], (ngu >> 1) & 1, kTagUnit, ngu, q)) break;
          const int cnt = hcount[hb];
          hcount[hb] = 0;
          if (cnt) {
            fence_proxy_async_global();
            red_release_gpu_add(p.tile_done + d.tile, cnt);
          }
          ++ngu;
        }
        mbar_arrive(&uempty[us]);
      }
    }
  } else {
    // --------------------------------------------------- compute ---
    uint32_t si = 0;
    int ngu = 0;
    for (int j = 0;; ++j) {
      const int us = j % kDecUnitRing;
      if (!__all_sync(0xFFFFFFFFu, ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -2))) break;
      const int q = uent[us].x;
      __syncwarp();
      if (q < 0) {
        if (lane == 0) mbar_arrive(&uempty[us]);
        break;
      }
      const DecUnit d = decode_unit(p, q, n1, udesc[us]);
      const int gu = d.gemm == 0 ? ngu++ : -1;
      const bool ok =
          d.nr > 8 ? dec_unit<2, FMT>(p, d, smem, full, empty, ab, &uempty[us], &uent[us], hpub, hcount, gu, si, q, warp, lane)
                   : dec_unit<1, FMT>(p, d, smem, full, empty, ab, &uempty[us], &uent[us], hpub, hcount, gu, si, q, warp, lane);
      if (!ok) break;
    }
  }
  __syncthreads();
}

template <int FMT>
static cudaError_t launch_decode(const DecodeParams& p, int grid, const CUtensorMap (&tmc)[3],
                                 const CUtensorMap (&tms)[3], const CUtensorMap& tm_x, const CUtensorMap& tm_h,
                                 cudaStream_t s) {
  ProfileScope prof(FT_KERNEL_FFN_DECODE, s);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ffn_decode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kDecSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(ffn_decode_kernel<FMT>, dim3(grid), dim3(kDecThreads), kDecSmemBytes, s, p, tmc[0], tms[0], tmc[1],
                    tms[1], tmc[2], tms[2], tm_x, tm_h);
}

}  // namespace ftmoe
