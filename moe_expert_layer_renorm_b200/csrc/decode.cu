// Expert FFN, decode variant: a weight-streaming grouped GEMV/GEMM for groups
// of at most 16 token rows, bound by the NVFP4 weight bytes read from HBM.
//
// Why not tcgen05 here: with a handful of token rows per expert the MMA is
// a tall-skinny product, and every tcgen05.mma instruction consumes at most
// 128 (M side) x 16 (K) weights per ~100 cycles of its SM when the weights are
// the M operand; as the N operand (256 x 16 per instruction) the dequantised
// tile must be written to and read back from shared memory, which saturates
// its bandwidth first.  Streaming at HBM rate needs ~35 weights per clock per
// SM, so the weights instead flow from TMA-staged shared memory through
// registers straight into warp-level MMA fragments (mma.sync m16n8k16, f16 x
// f16 -> fp32): 256 weights per instruction, no shared-memory round trip for
// the dequantised values, and the tensor cores do the FMAs.
//
// CTA tile: 256 weight rows (16 compute warps x 16 rows) x all of the unit's K,
// for one expert's group of <= 16 token rows (two n = 8 MMA tiles).  A stage
// holds one matrix's 256 rows for 256 K plus the token rows for that K, so
// the gate/up GEMM alternates gate and up stages.
//   warp 0     TMA: codes (256 rows x 128 B, 128-byte swizzle) and scales
//              (256 rows x 16 B) of one matrix, 256 K per stage
//   warp 1     TMA: the group's 16 token rows for the same 256 K (16-row tiles
//              of the permuted f16 activations, or of h)
//   warps 2-17 compute: warp w owns rows 16w .. 16w + 15 of the tile
//
// K permutation.  A dot product may visit K in any order as long as both
// operands use the same order.  For MMA i (0..7) of a 128-K half stage,
// thread t of each quad supplies logical k in {2t, 2t+1, 2t+8, 2t+9}; they are
// mapped to physical k = 32 t + 4 i + {0, 1, 2, 3}.  So a thread's weights for
// all eight MMAs are 32 consecutive K of its row (one 16-byte load of codes,
// two scale bytes), and its token values are 32 consecutive K of the token row
// (four 16-byte loads).
#include <cuda.h>
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

constexpr int kDecThreads = 18 * 32;
constexpr int kDecRows = 256;      // weight rows per CTA tile
constexpr int kDecBN = 16;         // token rows per unit
constexpr int kDecStageK = 256;

template <int NMAT, int STAGES>
struct DecCfg {
  static constexpr int kCodes = kDecRows * 128;                      // 256 rows x 128 B of codes
  static constexpr int kWStageBytes = kCodes + kDecRows * 16;        // + 256 rows x 16 B of scales
  static constexpr int kBBoxBytes = kDecBN * 128;                    // 64 K x 16 rows of f16
  static constexpr int kBStageBytes = 4 * kBBoxBytes;                // 256 K
  static constexpr int kStageBytes = kWStageBytes + kBStageBytes;    // multiple of 1024
  static constexpr int kSmemBytes = 1024 + STAGES * kStageBytes + 2 * STAGES * 8 + 64;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void mma_f16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int NMAT, int STAGES>
__global__ void __launch_bounds__(kDecThreads, 1)
ffn_decode_kernel(const FfnParams p, const __grid_constant__ CUtensorMap tm_codes0,
                  const __grid_constant__ CUtensorMap tm_scales0, const __grid_constant__ CUtensorMap tm_codes1,
                  const __grid_constant__ CUtensorMap tm_scales1, const __grid_constant__ CUtensorMap tm_act) {
  using Cfg = DecCfg<NMAT, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);
  uint64_t* empty = full + STAGES;
  int* abort_flag = reinterpret_cast<int*>(empty + STAGES);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 2); mbar_init(&empty[i], 16); }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_codes0); prefetch_tmap(&tm_scales0);
    if (NMAT > 1) { prefetch_tmap(&tm_codes1); prefetch_tmap(&tm_scales1); }
  }
  if (warp == 1 && lane == 0) prefetch_tmap(&tm_act);
  __syncthreads();
  const Abort ab{abort_flag};
  const int n_units = *p.num_units;

  auto unit_range = [&](int u, int& e, int& mt, int& rb, int& nr, int& ws0, int& ws1) {
    const int4 d = p.units[u];
    e = d.x; mt = d.y; rb = d.z; nr = d.w & 0xFFFF;
    const int split = d.w >> 16;
    ws0 = split * p.stages_per_split;
    ws1 = min(p.nkw, ws0 + p.stages_per_split);
  };

  if (warp == 0) {
    // ------------------------------------------------ weight TMA ---
    if (lane == 0) {
      const CUtensorMap* tmc[2] = {&tm_codes0, &tm_codes1};
      const CUtensorMap* tms[2] = {&tm_scales0, &tm_scales1};
      uint32_t si = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int e, mt, rb, nr, ws0, ws1;
        unit_range(u, e, mt, rb, nr, ws0, ws1);
        const int slot = __ldg(p.slot_table + e);
        for (int ws = ws0; ws < ws1 && ok; ++ws)
          for (int m = 0; m < NMAT; ++m, ++si) {
            const int s = si % STAGES;
            if (!(ok = ab.wait(&empty[s], ((si / STAGES) & 1) ^ 1, kTagWEmpty, si, u))) break;
            mbar_arrive_expect_tx(&full[s], Cfg::kWStageBytes);
            uint8_t* st = smem + s * Cfg::kStageBytes;
            tma_load_3d(st, tmc[m], &full[s], ws * 128, mt * kDecRows, slot);
            tma_load_3d(st + Cfg::kCodes, tms[m], &full[s], ws * 16, mt * kDecRows, slot);
          }
      }
      for (uint32_t j = (si > STAGES ? si - STAGES : 0); j < si; ++j) {   // drain
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % STAGES], (j / STAGES) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- token TMA ---
    if (lane == 0) {
      uint32_t si = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int e, mt, rb, nr, ws0, ws1;
        unit_range(u, e, mt, rb, nr, ws0, ws1);
        for (int q = ws0 * NMAT; q < ws1 * NMAT; ++q, ++si) {
          const int ws = q / NMAT;
          const int s = si % STAGES;
          if (!(ok = ab.wait(&empty[s], ((si / STAGES) & 1) ^ 1, kTagBEmpty, si, u))) break;
          mbar_arrive_expect_tx(&full[s], Cfg::kBStageBytes);
          uint8_t* bst = smem + s * Cfg::kStageBytes + Cfg::kWStageBytes;
#pragma unroll
          for (int bx = 0; bx < 4; ++bx)
            tma_load_2d(bst + bx * Cfg::kBBoxBytes, &tm_act, &full[s], ws * kDecStageK + bx * 64, rb);
        }
      }
      for (uint32_t j = (si > STAGES ? si - STAGES : 0); j < si; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % STAGES], (j / STAGES) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
      }
    }
  } else {
    // --------------------------------------------------- compute ---
    const int cw = warp - 2;                 // 0..15
    const int g = lane >> 2, t = lane & 3;   // mma quad layout
    const int r_lo = 16 * cw + g;            // rows of the 256-row tile
    const int r_hi = r_lo + 8;
    uint32_t si = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      int e, mt, rb, nr, ws0, ws1;
      unit_range(u, e, mt, rb, nr, ws0, ws1);
      const int ntiles = (nr + 7) >> 3;      // 1 or 2
      float acc[NMAT][2][4];
#pragma unroll
      for (int m = 0; m < NMAT; ++m)
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int i = 0; i < 4; ++i) acc[m][nt][i] = 0.0f;

      for (int q = ws0 * NMAT; q < ws1 * NMAT; ++q, ++si) {
        const int m = q % NMAT;
        const int s = si % STAGES;
          if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&full[s], (si / STAGES) & 1, kTagWFull, si, u)))) break;
        const uint8_t* st = smem + s * Cfg::kStageBytes;
        const uint8_t* bst = st + Cfg::kWStageBytes;
        // one matrix's 256 rows x 256 K against the unit's token rows
        auto stage_mma = [&](float (&am)[2][4]) {
          const int n0 = g, n1 = 8 + g;   // token rows of MMA tiles 0 and 1
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint8_t* bbox = bst + (2 * h + (t >> 1)) * Cfg::kBBoxBytes;
            const int chunk = 4 * h + t;   // 16-byte chunk of the 128-byte row: 32 codes
            const uint4 clo = *reinterpret_cast<const uint4*>(st + r_lo * 128 + ((chunk ^ (r_lo & 7)) << 4));
            const uint4 chi = *reinterpret_cast<const uint4*>(st + r_hi * 128 + ((chunk ^ (r_hi & 7)) << 4));
            const uint8_t* sc = st + Cfg::kCodes;
            const uint32_t slo = *reinterpret_cast<const uint16_t*>(sc + r_lo * 16 + 8 * h + 2 * t);
            const uint32_t shi = *reinterpret_cast<const uint16_t*>(sc + r_hi * 16 + 8 * h + 2 * t);
            const uint32_t wlo[4] = {clo.x, clo.y, clo.z, clo.w};
            const uint32_t whi[4] = {chi.x, chi.y, chi.z, chi.w};
            // the thread's 32 K span two 16-K scale blocks: MMAs 0..3 and 4..7
            const uint32_t sl2[2] = {e4m3_pair_to_f16x2(slo & 0xFFu), e4m3_pair_to_f16x2(slo >> 8)};
            const uint32_t sh2[2] = {e4m3_pair_to_f16x2(shi & 0xFFu), e4m3_pair_to_f16x2(shi >> 8)};
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {   // word wd: codes of MMAs 2 wd and 2 wd + 1
              // token values for those two MMAs: 16-byte chunk wd of the thread's 64 bytes
              const int cb = (t & 1) * 4 + wd;
              const uint4 b0 = *reinterpret_cast<const uint4*>(bbox + n0 * 128 + ((cb ^ (n0 & 7)) << 4));
              uint4 b1 = make_uint4(0u, 0u, 0u, 0u);
              if (ntiles > 1) b1 = *reinterpret_cast<const uint4*>(bbox + n1 * 128 + ((cb ^ (n1 & 7)) << 4));
              const uint32_t sl = sl2[wd >> 1], sh = sh2[wd >> 1];
              uint32_t qlo[4], qhi[4];
              e2m1x8_to_f16x2(wlo[wd], qlo);
              e2m1x8_to_f16x2(whi[wd], qhi);
              {
                const uint32_t a0 = hmul2_f16(qlo[0], sl), a1 = hmul2_f16(qhi[0], sh);
                const uint32_t a2 = hmul2_f16(qlo[1], sl), a3 = hmul2_f16(qhi[1], sh);
                mma_f16_16816(am[0], a0, a1, a2, a3, b0.x, b0.y);
                if (ntiles > 1) mma_f16_16816(am[1], a0, a1, a2, a3, b1.x, b1.y);
              }
              {
                const uint32_t a0 = hmul2_f16(qlo[2], sl), a1 = hmul2_f16(qhi[2], sh);
                const uint32_t a2 = hmul2_f16(qlo[3], sl), a3 = hmul2_f16(qhi[3], sh);
                mma_f16_16816(am[0], a0, a1, a2, a3, b0.z, b0.w);
                if (ntiles > 1) mma_f16_16816(am[1], a0, a1, a2, a3, b1.z, b1.w);
              }
            }
          }
        };
        if (NMAT == 1 || m == 0) stage_mma(acc[0]);
        else stage_mma(acc[NMAT - 1]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      if (!ok) break;

      // ------------------------------------------------ epilogue ---
      const int slot = __ldg(p.slot_table + e);
      const uint8_t* sbase = p.pool + size_t(slot) * size_t(p.slot_bytes);
      float gsc[NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) gsc[m] = __ldg(reinterpret_cast<const float*>(sbase + p.global_off[m]));
      const int f0 = mt * kDecRows + r_lo;   // features of c0/c1 (f0) and c2/c3 (f0 + 8)
      if (p.splits > 1) {
        // partials[u][m][n][256 rows]
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int n = 8 * nt + 2 * t + (i & 1);
              const int rr = r_lo + (i >> 1) * 8;
              if (n < nr) p.partials[((size_t(u) * NMAT + m) * kDecBN + n) * kDecRows + rr] = acc[m][nt][i];
            }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(p.counters + (u / p.splits) * 16 + cw, 1) == p.splits - 1;
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (!last) continue;
        __threadfence();
        const int u0 = u - (p.units[u].w >> 16);
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int n = 8 * nt + 2 * t + (i & 1);
              const int rr = r_lo + (i >> 1) * 8;
              float a = 0.0f;
              if (n < nr)
                for (int sp = 0; sp < p.splits; ++sp)
                  a += __ldcg(p.partials + ((size_t(u0 + sp) * NMAT + m) * kDecBN + n) * kDecRows + rr);
              acc[m][nt][i] = a;
            }
        if (lane == 0) p.counters[(u / p.splits) * 16 + cw] = 0;
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = 8 * nt + 2 * t + (i & 1);
          const int f = f0 + (i >> 1) * 8;
          if (n < nr && f < p.M) {
            float r;
            if (NMAT == 2) {
              const float ts = token_factor(p, rb + n);
              r = silu_mul(gsc[0] * ts * acc[0][nt][i], gsc[NMAT - 1] * ts * acc[NMAT - 1][nt][i]);
            } else {
              r = gsc[0] * acc[0][nt][i];
            }
            store_out<NMAT>(p.out, size_t(rb + n) * p.M + f, r);
          }
        }
    }
  }
  __syncthreads();
}

template <int NMAT, int STAGES>
static cudaError_t launch_decode_gemm(const FfnParams& p, int grid, const CUtensorMap& c0, const CUtensorMap& s0,
                                      const CUtensorMap& c1, const CUtensorMap& s1, const CUtensorMap& act,
                                      cudaStream_t s) {
  using Cfg = DecCfg<NMAT, STAGES>;
  ProfileScope prof(NMAT == 2 ? FT_KERNEL_GEMM_GATE_UP : FT_KERNEL_GEMM_DOWN, s);
  auto kern = ffn_decode_kernel<NMAT, STAGES>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<grid, kDecThreads, Cfg::kSmemBytes, s>>>(p, c0, s0, c1, s1, act);
  return cudaGetLastError();
}

}  // namespace ftmoe
