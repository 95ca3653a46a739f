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
// Work units (built on the device by ffn_schedule_kernel), in one queue:
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
// CTA (18 warps):
//   warps 0-15  compute, as 4 row groups x 4 K groups: warp w owns rows
//               64 (w & 3) .. +63 of the 256-row tile and K 64 (w >> 2) .. +63
//               of each 256-K stage, so a token value is read from shared
//               memory by 4 warps (not 16).  At the end of a unit the four
//               K-group warps of a row group exchange partial sums through
//               shared memory so that each owns a quarter of the outputs,
//               summed over K groups in a fixed order (deterministic), and
//               runs the epilogue for it.
//   warp 16     takes units from the queue; TMA of the 256 weight rows (two
//               128-row boxes of codes, 128-byte swizzle, and of scales)
//   warp 17     TMA of the unit's token rows (16-row boxes of the permuted f16
//               activations or of h), after the dependency wait for down units
//
// K permutation.  A dot product may visit K in any order as long as both
// operands use the same order.  Thread t of each quad supplies logical k in
// {2t, 2t+1, 2t+8, 2t+9} of MMA step i (0..3) of its 64-K slice; they are
// mapped to physical k = 16 t + 4 i + {0, 1, 2, 3}.  So a thread's 16 K of a
// row are one 16-element NVFP4 scale block (one 8-byte load of codes, one
// scale byte), and its token values are 16 consecutive K (two 16-byte loads).
#include <cuda.h>
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

constexpr int kDecThreads = 18 * 32;
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
constexpr int kDecRedBytes = 4 * 3 * 4 * 2 * 32 * 16;     // owner quarter x 3 sources x row groups x n-tiles x lanes
constexpr int kDecSmemBytes =
    1024 + kDecStages * kDecStageBytes + kDecRedBytes + (2 * kDecStages + 2 * kDecUnitRing + 2) * 8 + 64;
constexpr int kDecPartialBytes = 4 * 4 * 2 * 32 * 16;     // one unit's split-K partial sums (row group x quarter x n-tile x lane)
static_assert(kDecStageBytes % 1024 == 0, "stage alignment");
static_assert(kDecSmemBytes <= 227 * 1024, "shared memory budget");

// Barrier tag of the down unit's wait for its h rows.
constexpr int kTagDep = 9;

struct DecodeParams {
  FfnParams g[2];      // [0] gate/up + SwiGLU (h out), [1] down (out_perm out)
  int* queue;          // next queue position to take (zeroed by ffn_schedule_kernel)
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

__device__ __forceinline__ DecUnit decode_unit(const DecodeParams& p, int q, int n1) {
  DecUnit d;
  d.gemm = q < n1 ? 0 : 1;
  d.u = d.gemm ? q - n1 : q;
  const FfnParams& g = p.g[d.gemm];
  const int4 v = g.units[d.u];
  d.e = v.x & 1023; d.slot = v.x >> 10;
  d.mt = v.y; d.rb = v.z; d.nr = v.w & 0xFFFF;
  d.split = v.w >> 16;
  d.ws0 = d.split * g.stages_per_split;
  d.ws1 = min(g.nkw, d.ws0 + g.stages_per_split);
  const int per_tile = (d.gemm ? p.mt2 : p.mt1) * g.splits;
  d.tile = d.u / per_tile;
  return d;
}

// Stage-relative row of m-tile j (16 rows) of row group mg.  Gate/up stages
// hold the 128 gate rows then the 128 up rows of the same features; row group
// mg takes gate features 32 mg .. +31 (m-tiles 0, 1) and the up rows of the
// same features (m-tiles 2, 3), so one thread ends up with both halves of
// each SwiGLU.  Down stages: rows 64 mg + 16 j.
__device__ __forceinline__ int dec_row_base(int gemm, int mg, int j) {
  return gemm ? 64 * mg + 16 * j : (j < 2 ? 32 * mg + 16 * j : kDecFeat1 + 32 * mg + 16 * (j - 2));
}

// One 256-K stage for this warp: its 64 rows (4 m-tiles) x its 64 K x NT
// token tiles of 8.
template <int NT>
__device__ __forceinline__ void dec_stage(const uint8_t* st, const int (&rlo)[4], int kg, int g, int t,
                                          float (&acc)[4][NT][4]) {
  const uint8_t* bbox = st + kDecWStageBytes + kg * kDecBBoxBytes;
  uint4 bt[NT][2];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const int row = 8 * n + g;   // token row; its 16 K are 16-byte chunks 2t, 2t+1 (swizzled)
    bt[n][0] = *reinterpret_cast<const uint4*>(bbox + row * 128 + (((2 * t) ^ (row & 7)) << 4));
    bt[n][1] = *reinterpret_cast<const uint4*>(bbox + row * 128 + (((2 * t + 1) ^ (row & 7)) << 4));
  }
  const int cchunk = 2 * kg + (t >> 1), cbyte = 8 * (t & 1);
  const uint8_t* sc = st + kDecCodes + 4 * kg + t;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int rl = rlo[j], rh = rl + 8;
    const uint2 clo = *reinterpret_cast<const uint2*>(st + rl * 128 + ((cchunk ^ (rl & 7)) << 4) + cbyte);
    const uint2 chi = *reinterpret_cast<const uint2*>(st + rh * 128 + ((cchunk ^ (rh & 7)) << 4) + cbyte);
    const uint32_t sl = e4m3_pair_to_f16x2(sc[rl * 16]);
    const uint32_t sh = e4m3_pair_to_f16x2(sc[rh * 16]);
    uint32_t ql[2][4], qh[2][4];
    e2m1x8_to_f16x2(clo.x, ql[0]);
    e2m1x8_to_f16x2(clo.y, ql[1]);
    e2m1x8_to_f16x2(chi.x, qh[0]);
    e2m1x8_to_f16x2(chi.y, qh[1]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {   // physical k 16t + 4i + {0,1} (a0/a1, b0) and + {2,3} (a2/a3, b1)
      const int w = i >> 1, o = (i & 1) * 2;
      const uint32_t a0 = hmul2_f16(ql[w][o], sl), a1 = hmul2_f16(qh[w][o], sh);
      const uint32_t a2 = hmul2_f16(ql[w][o + 1], sl), a3 = hmul2_f16(qh[w][o + 1], sh);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const uint4& b = bt[n][i >> 1];
        mma_f16_16816(acc[j][n], a0, a1, a2, a3, (i & 1) ? b.z : b.x, (i & 1) ? b.w : b.y);
      }
    }
  }
}

// Output quarters.  After the main loop the four K-group warps of a row group
// split the row group's outputs four ways: warp kg owns quarter kg, i.e.
// m-tiles p = kg & 1 and p + 2, fragment half hh = kg >> 1 (rows g + 8 hh),
// every token tile.  For gate/up that is gate and up of the same features (a
// whole SwiGLU); for down, two 16-row m-tiles.  Per token tile a quarter is
// one float4: {m-tile p: token 2t, 2t+1;  m-tile p+2: token 2t, 2t+1}.
template <int NT>
__device__ __forceinline__ float4 dec_quarter(const float (&acc)[4][NT][4], int qq, int n) {
  const int p = qq & 1, hh = qq >> 1;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int pp = 0; pp < 2; ++pp)
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2)
      if (pp == p && h2 == hh)
        v = make_float4(acc[pp][n][2 * h2], acc[pp][n][2 * h2 + 1], acc[pp + 2][n][2 * h2], acc[pp + 2][n][2 * h2 + 1]);
  return v;
}

__device__ __forceinline__ void add4(float4& a, const float4& b) { a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w; }

// Epilogue of warp (mg, kg) for its quarter, once `v` holds the CTA's sums.
// With split-K across CTAs the quarter is first left as a partial sum; the
// last split to arrive adds all splits in order and finishes.
// Per-unit epilogue constants, loaded when the unit starts so that their
// latency hides behind the main loop.
struct DecConsts {
  float g0, g1;        // global scales: gate and up (gate/up unit) or down twice
  int any_scaled;      // gate/up: some token row was prescaled to fit f16
};

__device__ __forceinline__ DecConsts dec_consts(const DecodeParams& p, const DecUnit& d) {
  const FfnParams& G = p.g[d.gemm];
  const uint8_t* sbase = G.pool + size_t(d.slot) * size_t(G.slot_bytes);
  DecConsts c;
  c.g0 = __ldg(reinterpret_cast<const float*>(sbase + G.global_off[0]));
  c.g1 = __ldg(reinterpret_cast<const float*>(sbase + G.global_off[1]));
  c.any_scaled = d.gemm == 0 ? *G.any_scaled : 0;
  return c;
}

template <int NT>
__device__ __forceinline__ void dec_epilogue(const DecodeParams& p, const DecUnit& d, const DecConsts& c, int mg,
                                             int kg, int lane, float4 (&v)[NT]) {
  const FfnParams& G = p.g[d.gemm];
  const int g = lane >> 2, t = lane & 3;
  if (G.splits > 1) {
    // leave the partial quarter; the last split to arrive (acquire) sums them
    float4* part = reinterpret_cast<float4*>(G.partials);
    constexpr int kPer = kDecPartialBytes / 16;
    const int slot = ((mg * 4 + kg) * 2) * 32 + lane;
#pragma unroll
    for (int n = 0; n < NT; ++n) part[size_t(d.u) * kPer + slot + n * 32] = v[n];
    __syncwarp();
    int last = 0;
    if (lane == 0)
      last = atom_acq_rel_gpu_add(G.counters + (d.u / G.splits) * 16 + mg * 4 + kg, 1) == G.splits - 1;
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (!last) return;
    const int u0 = d.u - d.split;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < G.splits; ++sp)   // fixed order: the same sums whoever arrives last
        add4(s, __ldcg(part + size_t(u0 + sp) * kPer + slot + n * 32));
      v[n] = s;
    }
  }
  const int pq = kg & 1, hh = kg >> 1;
  if (d.gemm == 0) {
    const float gs = c.g0, gu = c.g1;
    const int f = d.mt * kDecFeat1 + 32 * mg + 16 * pq + g + 8 * hh;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 8 * n + 2 * t + e;
        if (r < d.nr && f < G.M) {
          const float ts = c.any_scaled ? __ldg(G.tokscale + __ldg(G.perm_src + d.rb + r) / G.k_top) : 1.0f;
          const float gv = e ? v[n].y : v[n].x, uv = e ? v[n].w : v[n].z;
          store_out<2>(G.out, size_t(d.rb + r) * G.M + f, silu_mul(gs * ts * gv, gu * ts * uv));
        }
      }
    // publish (release, after the warp's stores; the reader acquires the count
    // and orders its TMA reads behind it with a proxy fence)
    fence_proxy_async_global();
    __syncwarp();
    if (lane == 0) red_release_gpu_add(p.tile_done + d.tile, 1);
  } else {
    const float gd = c.g0;
    const int f = d.mt * kDecRows + 64 * mg + 16 * pq + g + 8 * hh;
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = 8 * n + 2 * t + e;
        if (r < d.nr) {
          float* o = static_cast<float*>(G.out) + size_t(d.rb + r) * G.M;
          if (f < G.M) o[f] = gd * (e ? v[n].y : v[n].x);
          if (f + 32 < G.M) o[f + 32] = gd * (e ? v[n].w : v[n].z);
        }
      }
  }
}

// Barrier tags of the unit ring and of the K-group hand-off.
constexpr int kTagUnit = 10;
constexpr int kTagRed = 11;

struct DecBars {
  uint64_t* full;      // [kDecStages]  weights + tokens of a stage landed (2 arrivals + bytes)
  uint64_t* empty;     // [kDecStages]  the 16 compute warps are done with a stage
  uint64_t* redfull;   // all 16 compute warps stored their partial quarters (512 threads)
  uint64_t* redfree;   // all 16 read theirs (512 threads)
};

// The main loop, K-group hand-off and epilogue of one unit for compute warp
// (mg, kg).  `si` counts stages consumed by this CTA, `j` units.  The unit's
// ring slot is released after the main loop, so a CTA takes a new unit from
// the queue only when it has finished computing the one before the current
// one: no CTA hoards small units while others idle.  Returns false if a wait
// gave up (the kernel then winds down).
template <int NT>
__device__ bool dec_unit(const DecodeParams& p, const DecUnit& d, uint8_t* smem, float4* red, const DecBars& b,
                         const Abort& ab, uint64_t* unit_free, const int4* unit_ent, uint32_t& si, int j, int q,
                         int mg, int kg, int lane) {
  const int g = lane >> 2, t = lane & 3;
  int rlo[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) rlo[jj] = dec_row_base(d.gemm, mg, jj) + g;
  float acc[4][NT][4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[jj][n][i] = 0.0f;

  for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
    const int s = si % kDecStages;
    if (!__all_sync(0xFFFFFFFFu, ab.wait(&b.full[s], (si / kDecStages) & 1, kTagWFull, si, q))) return false;
    dec_stage<NT>(smem + s * kDecStageBytes, rlo, kg, g, t, acc);
    __syncwarp();
    if (lane == 0) mbar_arrive(&b.empty[s]);
  }
  DecConsts c;   // written by the weight producer before the last stage (acquired above)
  {
    const int4 ce = *unit_ent;
    c.g0 = __int_as_float(ce.y); c.g1 = __int_as_float(ce.z); c.any_scaled = ce.w;
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(unit_free);   // the queue may hand this CTA its next-but-one unit

  // hand the other three quarters to their owners; red[owner][source][mg][n][lane]
  auto slot = [&](int owner, int src, int n) {
    return red + ((((owner * 3 + (src < owner ? src : src - 1)) * 4 + mg) * 2 + n) * 32 + lane);
  };
  if (j > 0 && !__all_sync(0xFFFFFFFFu, ab.wait(b.redfree, (j - 1) & 1, kTagRed, j, q))) return false;
#pragma unroll
  for (int qq = 0; qq < 4; ++qq)
    if (qq != kg)
#pragma unroll
      for (int n = 0; n < NT; ++n) *slot(qq, kg, n) = dec_quarter<NT>(acc, qq, n);
  mbar_arrive(b.redfull);
  if (!__all_sync(0xFFFFFFFFu, ab.wait(b.redfull, j & 1, kTagRed, j, q))) return false;
  float4 v[NT];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    v[n] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int src = 0; src < 4; ++src)   // K groups in order: deterministic sums
      add4(v[n], src == kg ? dec_quarter<NT>(acc, kg, n) : *slot(kg, src, n));
  }
  mbar_arrive(b.redfree);
  dec_epilogue<NT>(p, d, c, mg, kg, lane, v);
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

__global__ void __launch_bounds__(kDecThreads, 1)
ffn_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_c0,
                  const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_c1,
                  const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_c2,
                  const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_h) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float4* red = reinterpret_cast<float4*>(smem + kDecStages * kDecStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecStages * kDecStageBytes + kDecRedBytes);
  DecBars b{bars, bars + kDecStages, bars + 2 * kDecStages + 2 * kDecUnitRing,
            bars + 2 * kDecStages + 2 * kDecUnitRing + 1};
  uint64_t* ufull = bars + 2 * kDecStages;
  uint64_t* uempty = ufull + kDecUnitRing;
  // ring entries: {queue position, then (before the unit's last stage lands)
  // the epilogue constants: global scale bits x2, any token prescaled}
  int4* uent = reinterpret_cast<int4*>(bars + 2 * kDecStages + 2 * kDecUnitRing + 2);
  int* abort_flag = reinterpret_cast<int*>(uent + kDecUnitRing);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecStages; ++i) { mbar_init(&b.full[i], 2); mbar_init(&b.empty[i], 16); }
    for (int i = 0; i < kDecUnitRing; ++i) { mbar_init(&ufull[i], 1); mbar_init(&uempty[i], 17); }
    mbar_init(b.redfull, 512);
    mbar_init(b.redfree, 512);
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
      for (int j = 0; ok; ++j) {
        const int us = j % kDecUnitRing;   // take a unit only once there is room to hold it
        if (!(ok = ab.wait(&uempty[us], ((j / kDecUnitRing) & 1) ^ 1, kTagUnit, j, -3))) break;
        int q = atomicAdd(p.queue, 1);
        if (q >= ntot) q = -1;
        uent[us].x = q;
        mbar_arrive(&ufull[us]);
        if (q < 0) break;
        const DecUnit d = decode_unit(p, q, n1);
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
          if (!(ok = ab.wait(&b.empty[s], ((si / kDecStages) & 1) ^ 1, kTagWEmpty, si, q))) break;
          if (ws == d.ws1 - 1)   // published by this stage's arrival (release) to the compute warps
            uent[us] = make_int4(q, __float_as_int(c.g0), __float_as_int(c.g1), c.any_scaled);
          mbar_arrive_expect_tx(&b.full[s], kDecWStageBytes);
          uint8_t* st = smem + s * kDecStageBytes;
          tma_load_3d(st, c0, &b.full[s], ws * 128, y0, slot);
          tma_load_3d(st + 128 * 128, c1, &b.full[s], ws * 128, y1, slot);
          tma_load_3d(st + kDecCodes, s0, &b.full[s], ws * 16, y0, slot);
          tma_load_3d(st + kDecCodes + 128 * 16, s1, &b.full[s], ws * 16, y1, slot);
        }
      }
      dec_drain(b.full, si);
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
        const DecUnit d = decode_unit(p, q, n1);
        if (d.gemm == 1) {
          if (!(ok = dec_wait_h(p, d, ab, q))) break;
          fence_proxy_async_global();   // the h rows were written by generic stores
        }
        const CUtensorMap* act = d.gemm ? &tm_h : &tm_x;
        for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
          const int s = si % kDecStages;
          if (!(ok = ab.wait(&b.empty[s], ((si / kDecStages) & 1) ^ 1, kTagBEmpty, si, q))) break;
          mbar_arrive_expect_tx(&b.full[s], kDecBStageBytes);
          uint8_t* bst = smem + s * kDecStageBytes + kDecWStageBytes;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_2d(bst + bx * kDecBBoxBytes, act, &b.full[s], ws * kDecStageK + bx * 64, d.rb);
        }
        mbar_arrive(&uempty[us]);
      }
      dec_drain(b.full, si);
    }
  } else {
    // --------------------------------------------------- compute ---
    const int mg = warp & 3, kg = warp >> 2;
    uint32_t si = 0;
    for (int j = 0;; ++j) {
      const int us = j % kDecUnitRing;
      if (!__all_sync(0xFFFFFFFFu, ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -2))) break;
      const int q = uent[us].x;
      __syncwarp();
      if (q < 0) {
        if (lane == 0) mbar_arrive(&uempty[us]);
        break;
      }
      const DecUnit d = decode_unit(p, q, n1);
      const bool ok = d.nr > 8 ? dec_unit<2>(p, d, smem, red, b, ab, &uempty[us], &uent[us], si, j, q, mg, kg, lane)
                               : dec_unit<1>(p, d, smem, red, b, ab, &uempty[us], &uent[us], si, j, q, mg, kg, lane);
      if (!ok) break;
    }
  }
  __syncthreads();
}

static cudaError_t launch_decode(const DecodeParams& p, int grid, const CUtensorMap (&tmc)[3],
                                 const CUtensorMap (&tms)[3], const CUtensorMap& tm_x, const CUtensorMap& tm_h,
                                 cudaStream_t s) {
  ProfileScope prof(FT_KERNEL_FFN_DECODE, s);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(ffn_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kDecSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  ffn_decode_kernel<<<grid, kDecThreads, kDecSmemBytes, s>>>(p, tmc[0], tms[0], tmc[1], tms[1], tmc[2], tms[2],
                                                             tm_x, tm_h);
  return cudaGetLastError();
}

}  // namespace ftmoe
