// Expert FFN over permuted rows: a grouped GEMM with NVFP4 weights on tcgen05.
//
// Orientation ("swap AB"): the MMA's M side (128 rows) is 128 output features
// of one expert's weight matrix and its N side is up to BN permuted token
// rows of that expert's group, so any group size from 1 row up maps onto one
// instruction shape (N = group rows rounded up to 16).
//
// Data path of one CTA (persistent; 16 warps), per KC-wide chunk of K:
//   warp 0      TMA: packed E2M1 codes (128 rows x 128 B, 128-byte swizzle)
//               and E4M3 scales (128 rows x 16 B) of each matrix, 256 K per stage
//   warp 2      TMA: the unit's token rows (f16) into 128-byte-swizzled K-major
//               shared memory (the MMA's B operand): one BN-row box per 64-K
//               swizzle atom, of the permuted f16 activations (GEMM1) or of h
//               (GEMM2); both are stored in permuted row order
//   warps 4-11  two warpgroups, alternate chunks: E2M1 -> f16 (cvt) times the
//               E4M3 block scale (exact in f16), stored with tcgen05.st
//               straight into tensor memory, where the MMA reads it as its A
//               operand (no shared-memory round trip)
//   warp 3      waits on the operand barriers for the MMA warp and hands each
//               ready chunk over at a named barrier
//   warp 1      one thread issues tcgen05.mma kind::f16 (f16 x f16 -> fp32
//               accumulators in tensor memory) and commits to the barriers;
//               it waits on no mbarrier inside its loop
//   warps 12-15 epilogue: tcgen05.ld of the accumulators, fp32 global scale,
//               SwiGLU (GEMM1) and f16 h / fp32 output stores; for split-K,
//               fp32 partials and a last-arriving-CTA reduction in a fixed
//               order (deterministic)
//
// Every pipeline wait is bounded (see sm100.cuh); a wait that gives up sets
// the device status word and an abort flag, all roles leave their loops, and
// the CTA drains its outstanding copies and MMAs before freeing tensor memory.
#include <type_traits>

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

constexpr int kKW = 256;            // K per weight stage (128 bytes of codes per row)
constexpr int kAtomK = 64;          // K of one 128-byte swizzle atom of f16 (one token-tile box)
constexpr int kCodesBytes = 128 * 128;
constexpr int kScaleBytes = 128 * 16;
constexpr int kMatStageBytes = kCodesBytes + kScaleBytes;   // 18 KB, multiple of 1024
constexpr int kThreads = 512;

struct FfnParams {
  const float* rowscale;      // per permuted row, its factor f_r = 2^e_r (see silu_mul); null reads as 1
  const int32_t* perm_src;    // GEMM1: row -> pair (token = pair / k_top); GEMM2: null (row -> row)
  int k_top;
  int K;                      // reduction length
  int M;                      // output features (rows of the weight matrices)
  int nkw;                    // ceil(K / kKW)
  int nkc;                    // ceil(K / KC): chunks of the kernel's chunk size
  int splits;                 // split-K factor
  int stages_per_split;
  const int4* units;          // {expert | slot << 10, m_tile, row_begin, n_rows | split << 16}
  const int* num_units;
  const int32_t* slot_table;
  const uint8_t* pool;
  long long slot_bytes;
  long long global_off[2];
  void* out;                  // GEMM1: h f16 [P, M]; GEMM2: out_perm fp32 [P, M]
  float* partials;            // split-K partial accumulators
  int* counters;              // split-K arrival counters, 4 per (tile, m_tile): one per epilogue warp
  int tiled;                  // weight maps are 4-D over stage-tiled slots (else 3-D over row-major ones)
};

// KC: K per chunk (64 or 128), the unit of one dequantised A slot, one
// token stage and one operand hand-over to the MMA warp.  A chunk of 128
// halves the per-chunk costs (barriers, hand-over, commits) per MMA.
// AM: where the dequantised A operand lives -- 0: tensor memory (the MMA's TS
// form, tcgen05.st from the dequantising warps), 1: shared memory (SS form,
// 128-byte-swizzled K-major rows like the token boxes), which leaves tensor
// memory to the accumulators.
template <int NMAT, int BN, int WS, int BS, int AS, int DB, int KC, int AM = 0>
struct FfnCfg {
  static constexpr int kAtoms = KC / kAtomK;                 // swizzle atoms (token boxes) per chunk
  static constexpr int kCPW = kKW / KC;                      // chunks per weight stage
  static constexpr int kACols = KC / 2;                      // tensor-memory columns of one matrix's A slot
  static constexpr int kWBytes = WS * NMAT * kMatStageBytes;
  static constexpr int kBAtomBytes = BN * 128;
  static constexpr int kBStageBytes = kAtoms * kBAtomBytes;
  static constexpr int kBBytes = BS * kBStageBytes;
  static constexpr int kAAtomBytes = 128 * 128;               // one 64-K atom of 128 weight rows, f16
  static constexpr int kABytes = AM ? AS * NMAT * kAtoms * kAAtomBytes : 0;
  static constexpr int kNumBars = 2 * WS + 2 * BS + 2 * AS + 2 * DB + 1;
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kWBytes + kBBytes + kABytes + BN * 4 + kNumBars * 8 + 64;
  static constexpr int kDCols = DB * NMAT * BN;
  static constexpr int kTmemCols = kDCols + (AM ? 0 : AS * NMAT * kACols);
  static_assert(KC == 64 || KC == 128, "chunk size");
  static_assert(kTmemCols <= 512, "tensor memory budget");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// ------------------------------------------------------------ dequant ---

__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t v, uint32_t (&q)[4]) {
  asm("{.reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3]) : "r"(v));
}
__device__ __forceinline__ uint32_t e4m3_pair_to_f16x2(uint32_t byte) {   // (s, s)
  uint32_t r;
  const uint16_t in = uint16_t(byte | (byte << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(in));
  return r;
}
// E8M0 scale byte s of an MXFP4 block -> (2^(s - bias), 2^(s - bias)) in f16,
// bias = 127 + t with 2^t the tensor's global: from the exponent bits (normal
// for s - bias >= -14, subnormal down to 2^-24, zero below; the pack keeps
// s - bias <= 13).
__device__ __forceinline__ uint32_t e8m0_pair_to_f16x2(uint32_t byte, int bias) {
  const int e = min(int(byte) - bias, 15);
  const uint32_t h = e >= -14 ? uint32_t(e + 15) << 10 : (e >= -24 ? 1u << (e + 24) : 0u);
  return h | (h << 16);
}
// The shift that the dequantisation takes out of MXFP4 scales: 127 + log2 of
// the tensor's global (a power of two).
__device__ __forceinline__ int mx_bias(float global) { return 127 + ilogbf(global); }

// Two E4M3 scale bytes (the low byte is the first block's) -> (s0, s0) and
// (s1, s1) in f16: one conversion and two byte permutes, about half the ALU
// instructions of converting each byte on its own (the decode kernel's inner
// loop is bound by the ALU pipe: measured 79.6 vs 82.0 us at decode_T64).
__device__ __forceinline__ void e4m3x2_to_pairs(uint32_t two, uint32_t& p0, uint32_t& p1) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(uint16_t(two)));
  p0 = __byte_perm(r, 0, 0x1010);
  p1 = __byte_perm(r, 0, 0x3232);
}

// Scale byte of one 16-K block -> f16x2 (s, s) in the slot's format.
template <int FMT>
__device__ __forceinline__ uint32_t scale_pair_to_f16x2(uint32_t byte, int bias) {
  if (FMT == FT_SCALE_MXFP4) return e8m0_pair_to_f16x2(byte, bias);
  return e4m3_pair_to_f16x2(byte);
}

__device__ __forceinline__ uint32_t hmul2_f16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
// f16x2 -> bf16x2 of the same values (exact for E2M1 x E4M3 products: at most
// 6 significant bits, magnitudes in [2^-10, 2688]).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h) {
  uint32_t r;
  asm("{.reg .b16 a, b;\n .reg .f32 fa, fb;\n mov.b32 {a, b}, %1;\n cvt.f32.f16 fa, a;\n"
      " cvt.f32.f16 fb, b;\n cvt.rn.bf16x2.f32 %0, fb, fa;\n}"
      : "=r"(r) : "r"(h));
  return r;
}

// 64 codes (two 16-byte words of one row) and their 4 scale bytes -> 32
// f16x2 words, word c holding k = 2c (low half) and 2c + 1 (high half).
// Every E2M1 x E4M3 product (at most 6 significant bits, magnitude in
// [2^-10, 2688]) is an exact f16, so the products carry no rounding.
template <int FMT>
__device__ __forceinline__ void dequant_chunk(const uint4& c0, const uint4& c1, uint32_t sc, int bias,
                                              uint32_t (&o)[32]) {
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  uint32_t sp[4];
  if (FMT == FT_SCALE_NVFP4) {
    e4m3x2_to_pairs(sc & 0xFFFFu, sp[0], sp[1]);
    e4m3x2_to_pairs(sc >> 16, sp[2], sp[3]);
  } else {
#pragma unroll
    for (int b = 0; b < 4; ++b) sp[b] = scale_pair_to_f16x2<FMT>((sc >> (8 * b)) & 0xFFu, bias);
  }
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    const uint32_t s2 = sp[b];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t q[4];
      e2m1x8_to_f16x2(w[2 * b + h], q);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[(2 * b + h) * 4 + j] = hmul2_f16(q[j], s2);
    }
  }
}

// ---------------------------------------------------------- pipeline ---

// Barrier kinds, recorded with a wait timeout.
enum : int { kTagWEmpty = 1, kTagWFull, kTagBEmpty, kTagBFull, kTagAEmpty, kTagAFull, kTagDEmpty, kTagDFull };

// Named barrier (id 0 is __syncthreads) shared by the MMA warp and the
// operand-waiter warp.
constexpr int kBarHandoff = 1;

struct Abort {
  volatile int* flag;
  __device__ bool wait(uint64_t* bar, uint32_t parity, int tag = 0, long long counter = 0,
                       long long unit = 0) const {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (true) {
      if (mbar_try_wait(bar, parity)) return true;
      if ((++n & 63u) == 0) {
        if (*flag) return false;
        const uint64_t dt = globaltimer_ns() - t0;
        if (dt > 1000000000ull) {
          set_device_status_detail(FT_DEV_WAIT_TIMEOUT, tag, counter, unit, (long long)(dt / 1000));
          *flag = 1;
          return false;
        }
      }
    }
  }
};

// Per-row normalisation of the token rows.  Row r (token t) has the
// exponent e_r (row_exp_of_max: 0 when max|x_t| is in [2, 8), else
// max|x_t| * 2^-e_r in [4, 8)), and rowscale[r] = f_r = 2^e_r.  GEMM1
// multiplies f16 operands x' = x * 2^(12 - e_r) (largest magnitude in
// [2^13, 2^15)), so with the global scale gG its accumulator gives
// G' = gG * 2^-12 * acc = G / f_r: the gate (and likewise the up) projection
// of the row scaled to a largest magnitude in [2, 8).  h is stored normalised
// the same way,
//   h' = silu(G) * U / f_r^2 = G' * U' / (1 + e^-(G' f_r)),
// so its f16 range does not depend on the row's magnitude, and GEMM2 undoes
// it exactly: out = (gD * acc * f_r) * f_r.  Rows of ordinary magnitude (the
// N(0, 1) workloads) have f_r = 1, and the epilogues skip the factor for
// units whose rows all have it.
constexpr float kRowNormInv = 1.0f / 4096.0f;   // 2^-12

// h' = g * u / (1 + e^-(g f)).  The hardware exponential and a fast divide: a
// few ulps of fp32, far inside the layer's tolerance; as g f -> -inf the
// divisor overflows to inf and the result goes to 0, its limit.
__device__ __forceinline__ float silu_mul(float g, float u, float f) {
  return __fdividef(g * u, 1.0f + __expf(-(g * f)));
}
// The same for f = 1.
__device__ __forceinline__ float silu_mul1(float g, float u) { return __fdividef(g * u, 1.0f + __expf(-g)); }
// GEMM2's output from its accumulator: (gD * acc * f) * f, in this order so
// that no intermediate leaves the fp32 range when the result does not.
__device__ __forceinline__ float down_out(float gd, float acc, float f) { return (gd * acc * f) * f; }

// GEMM1 stores h in f16 (it is the next MMA's operand; a value beyond the f16
// range saturates and records FT_DEV_F16_RANGE); GEMM2 stores the expert
// outputs in fp32 so that only the combine's own fp32 sum rounds them.
template <int NMAT>
__device__ __forceinline__ void store_out(void* out, size_t idx, float v) {
  if (NMAT == 2) {
    if (fabsf(v) > 65504.0f) {
      set_device_status(FT_DEV_F16_RANGE);
      v = copysignf(65504.0f, v);
    }
    static_cast<__half*>(out)[idx] = __float2half_rn(v);
  } else {
    static_cast<float*>(out)[idx] = v;
  }
}

// The row factor f_r of permuted row `row` (1 without a rowscale array).
__device__ __forceinline__ float token_factor(const FfnParams& p, int row) {
  return p.rowscale != nullptr ? __ldg(p.rowscale + row) : 1.0f;
}

template <int NMAT, int BN, int WS, int BS, int AS, int DB, int KC, int FMT, int AM>
__global__ void __launch_bounds__(kThreads, 1)
ffn_gemm_kernel(const FfnParams p, const __grid_constant__ CUtensorMap tm_codes0,
                const __grid_constant__ CUtensorMap tm_scales0, const __grid_constant__ CUtensorMap tm_codes1,
                const __grid_constant__ CUtensorMap tm_scales1, const __grid_constant__ CUtensorMap tm_act) {
  pdl_wait();   // dependents are triggered at the end (see below)
  using Cfg = FfnCfg<NMAT, BN, WS, BS, AS, DB, KC, AM>;
  constexpr int kCPW = Cfg::kCPW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* w_smem = smem;
  uint8_t* b_smem = smem + Cfg::kWBytes;
  uint8_t* a_smem = b_smem + Cfg::kBBytes;   // AM = 1: AS x NMAT x kAtoms atoms of 16 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(a_smem + Cfg::kABytes);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + WS;
  uint64_t* b_full = w_empty + WS;
  uint64_t* b_empty = b_full + BS;
  uint64_t* a_full = b_empty + BS;
  uint64_t* a_empty = a_full + AS;
  uint64_t* d_full = a_empty + AS;
  uint64_t* d_empty = d_full + DB;
  uint64_t* drain_bar = d_empty + DB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* handoff = abort_flag + 1;   // [2]: waiter -> MMA warp, per chunk (by parity): 1 go, 0 stop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < WS; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], 8); }
    for (int i = 0; i < BS; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < AS; ++i) { mbar_init(&a_full[i], 4); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < DB; ++i) { mbar_init(&d_full[i], 1); mbar_init(&d_empty[i], 4); }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_codes0); prefetch_tmap(&tm_scales0);
    if (NMAT > 1) { prefetch_tmap(&tm_codes1); prefetch_tmap(&tm_scales1); }
  }
  if (warp == 2 && lane == 0) prefetch_tmap(&tm_act);
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag};
  const int n_units = *p.num_units;
  const int nchunks_total = p.nkc;

  auto unit_range = [&](int u, int& e, int& mt, int& rb, int& nr, int& ws0, int& ws1, int& kc0, int& kc1) {
    const int4 d = p.units[u];
    e = d.x & 1023; mt = d.y; rb = d.z; nr = d.w & 0xFFFF;
    const int split = d.w >> 16;
    ws0 = split * p.stages_per_split;
    ws1 = min(p.nkw, ws0 + p.stages_per_split);
    kc0 = ws0 * kCPW;
    kc1 = min(nchunks_total, ws1 * kCPW);
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer ---
    uint32_t wi = 0;
    if (lane == 0) {
      const CUtensorMap* tmc[2] = {&tm_codes0, &tm_codes1};
      const CUtensorMap* tms[2] = {&tm_scales0, &tm_scales1};
      bool ok = true;
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int e, mt, rb, nr, ws0, ws1, kc0, kc1;
        unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
        const int slot = __ldg(p.slot_table + e);
        for (int ws = ws0; ws < ws1; ++ws, ++wi) {
          const int s = wi % WS;
          if (!(ok = ab.wait(&w_empty[s], ((wi / WS) & 1) ^ 1, kTagWEmpty, wi, u))) break;
          mbar_arrive_expect_tx(&w_full[s], NMAT * kMatStageBytes);
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            uint8_t* dst = w_smem + (s * NMAT + m) * kMatStageBytes;
            tma_load_weights(dst, tmc[m], &w_full[s], p.tiled, 128, ws, mt * 128, slot);
            tma_load_weights(dst + kCodesBytes, tms[m], &w_full[s], p.tiled, 16, ws, mt * 128, slot);
          }
        }
      }
      // drain: the last copy into every stage buffer has landed
      for (uint32_t j = (wi > WS ? wi - WS : 0); j < wi; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&w_full[j % WS], (j / WS) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA issuer ---
    // Waits on no mbarrier inside the loop: an mbarrier wait (or a polled
    // flag) in the issuing thread leaves the tensor pipe idle for a few
    // hundred cycles even when the operands are already in place.  Warp 3
    // does the waiting; the two warps meet at a named barrier once per chunk,
    // with warp 3 one chunk ahead, and warp 3 leaves its go or stop decision in
    // handoff[q & 1] before it arrives.  Both warps run the same chunk
    // sequence and leave at the same chunk, so every barrier phase completes.
    uint32_t q = 0, di = 0;
    bool ok = true, issued = false;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++di) {
      int e, mt, rb, nr, ws0, ws1, kc0, kc1;
      unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
      const int ds = di % DB;
      const int n_eff = (nr + 15) & ~15;
      const uint32_t idesc = make_idesc_f16(128, n_eff, /*f16 operands=*/true);
      for (int c = kc0; c < kc1; ++c, ++q) {
        named_bar_sync(kBarHandoff, 64);
        if (!(ok = *reinterpret_cast<volatile int*>(handoff + (q & 1)) != 0)) break;
        if (lane == 0) {
          tc_fence_after();
          const int as = q % AS, bs = q % BS;
          const uint64_t bd = make_sdesc_sw128(smem_u32(b_smem + bs * Cfg::kBStageBytes));
          const uint32_t d0 = tmem + ds * NMAT * BN;
          const uint32_t acc0 = c > kc0 ? 1u : 0u;
          if (AM) {   // A: atom (as, m, j / 4) of shared memory, +32 bytes per K slice in it
            const uint64_t ad = make_sdesc_sw128(smem_u32(a_smem + as * NMAT * Cfg::kAtoms * Cfg::kAAtomBytes));
#pragma unroll
            for (int j = 0; j < KC / 16; ++j)
#pragma unroll
              for (int m = 0; m < NMAT; ++m)
                mma_ss_f16(d0 + m * BN,
                           ad + uint64_t(((m * Cfg::kAtoms + j / 4) * Cfg::kAAtomBytes >> 4) + 2 * (j % 4)),
                           bd + uint64_t((j / 4) * (Cfg::kBAtomBytes >> 4) + 2 * (j % 4)), idesc,
                           j > 0 ? 1u : acc0);
          } else {
            const uint32_t a0 = tmem + Cfg::kDCols + as * NMAT * Cfg::kACols;
#pragma unroll
            for (int m = 0; m < NMAT; ++m) mma_ts_f16(d0 + m * BN, a0 + m * Cfg::kACols, bd, idesc, acc0);
#pragma unroll
            for (int j = 1; j < KC / 16; ++j)
#pragma unroll
              for (int m = 0; m < NMAT; ++m)   // K slice j: atom j / 4 (+kBAtomBytes), +32 bytes per slice in it
                mma_ts_f16_acc(d0 + m * BN, a0 + m * Cfg::kACols + 8 * j,
                               bd + uint64_t((j / 4) * (Cfg::kBAtomBytes >> 4) + 2 * (j % 4)), idesc);
          }
          mma_commit(&a_empty[as]);
          mma_commit(&b_empty[bs]);
        }
        issued = true;
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) mma_commit(&d_full[ds]);
      __syncwarp();
    }
    if (issued && lane == 0) {   // drain: every MMA this thread issued has completed
      mma_commit(drain_bar);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < 1000000000ull) {}
    }
  } else if (warp == 2) {
    // --------------------------------------------- B (token) producer ---
    // Lane 0 issues one BN-row TMA box per 64-K swizzle atom (one large box keeps
    // the copy engine's per-box cost off the critical path; 16-row boxes
    // were several times slower).  Rows past the group end are other
    // groups' rows (or zero fill past the last row): finite, and their
    // results are never stored.
    uint32_t q = 0;
    bool ok = true;
    if (lane == 0) {
      for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
        int e, mt, rb, nr, ws0, ws1, kc0, kc1;
        unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
        for (int c = kc0; c < kc1; ++c, ++q) {
          const int bs = q % BS;
          if (!(ok = ab.wait(&b_empty[bs], ((q / BS) & 1) ^ 1, kTagBEmpty, q, u))) break;
          mbar_arrive_expect_tx(&b_full[bs], uint32_t(Cfg::kBStageBytes));
#pragma unroll
          for (int a = 0; a < Cfg::kAtoms; ++a)   // K past the end reads as zeros (their A is zero too)
            tma_load_2d(b_smem + bs * Cfg::kBStageBytes + a * Cfg::kBAtomBytes, &tm_act, &b_full[bs],
                        c * KC + a * kAtomK, rb);
        }
      }
      for (uint32_t j = (q > BS ? q - BS : 0); j < q; ++j) {   // drain
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&b_full[j % BS], (j / BS) & 1) && globaltimer_ns() - t0 < 1000000000ull) {}
      }
    }
  } else if (warp == 3) {
    // ---------------------------------------------- operand waiter ---
    // Lane 0 waits, in the MMA warp's order, for each unit's accumulator
    // buffer to be drained and for each chunk's A (dequantised weights) and B
    // (tokens) to be in place; the warp then meets the MMA warp at the named
    // barrier.  Its place at warp index 3 also keeps the dequantising warps at
    // 4..11, so that warp % 4 names the 32-lane quarter of tensor memory each
    // of them may access.
    uint32_t q = 0, di = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++di) {
      int e, mt, rb, nr, ws0, ws1, kc0, kc1;
      unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
      const int ds = di % DB;
      for (int c = kc0; c < kc1; ++c, ++q) {
        if (lane == 0) {
          if (c == kc0) ok = ab.wait(&d_empty[ds], ((di / DB) & 1) ^ 1, kTagDEmpty, di, u);
          ok = ok && ab.wait(&a_full[q % AS], (q / AS) & 1, kTagAFull, q, u);
          ok = ok && ab.wait(&b_full[q % BS], (q / BS) & 1, kTagBFull, q, u);
          *reinterpret_cast<volatile int*>(handoff + (q & 1)) = ok ? 1 : 0;
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        named_bar_sync(kBarHandoff, 64);
        if (!ok) break;
      }
    }
  } else if (warp >= 4 && warp < 12) {
    // -------------------------------------------------- dequantise ---
    const int g = (warp - 4) >> 2;            // warpgroup: even / odd chunks
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;      // weight row within the tile = TMEM lane
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    uint32_t q = 0, wi = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x) {
      int e, mt, rb, nr, ws0, ws1, kc0, kc1;
      unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
      int bias[NMAT];   // MXFP4: the power of two the unit's globals take out of the scales
#pragma unroll
      for (int m = 0; m < NMAT; ++m) bias[m] = 0;
      if (FMT == FT_SCALE_MXFP4) {
        const uint8_t* sbase = p.pool + size_t(__ldg(p.slot_table + e)) * size_t(p.slot_bytes);
#pragma unroll
        for (int m = 0; m < NMAT; ++m) bias[m] = mx_bias(__ldg(reinterpret_cast<const float*>(sbase + p.global_off[m])));
      }
      for (int ws = ws0; ws < ws1 && ok; ++ws, ++wi) {
        const int s = wi % WS;
        if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&w_full[s], (wi / WS) & 1, kTagWFull, wi, u)))) break;
        const int c_end = min(kc1, (ws + 1) * kCPW);
        for (int c = ws * kCPW; c < c_end; ++c, ++q) {
          if ((q & 1) != uint32_t(g)) continue;
          const int as = q % AS;
          if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&a_empty[as], ((q / AS) & 1) ^ 1, kTagAEmpty, q, u)))) break;
          tc_fence_after();
          const int cc = c - ws * kCPW;
#pragma unroll
          for (int m = 0; m < NMAT; ++m) {
            const uint8_t* base = w_smem + (s * NMAT + m) * kMatStageBytes;
            const uint8_t* crow = base + row * 128;
#pragma unroll
            for (int h = 0; h < Cfg::kAtoms; ++h) {   // 64 K of the chunk: 16-byte words 2t, 2t + 1, scale word t
              const int t = cc * Cfg::kAtoms + h;
              const uint4 c0 = *reinterpret_cast<const uint4*>(crow + (((2 * t) ^ (row & 7)) << 4));
              const uint4 c1 = *reinterpret_cast<const uint4*>(crow + (((2 * t + 1) ^ (row & 7)) << 4));
              const uint32_t sc = *reinterpret_cast<const uint32_t*>(base + kCodesBytes + row * 16 + t * 4);
              uint32_t o[32];
              dequant_chunk<FMT>(c0, c1, sc, bias[m], o);
              if (AM) {   // row `row` of the atom, its eight 16-byte chunks 128-byte swizzled
                uint8_t* arow = a_smem + ((as * NMAT + m) * Cfg::kAtoms + h) * Cfg::kAAtomBytes + row * 128;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  *reinterpret_cast<uint4*>(arow + ((j ^ (row & 7)) << 4)) =
                      make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
              } else {
                tmem_st_32x32b_x32(tmem + lane_base + Cfg::kDCols + (as * NMAT + m) * Cfg::kACols + h * 32, o);
              }
            }
          }
          if (AM) {
            fence_proxy_async_smem();   // the generic stores, visible to the MMA's operand reads
          } else {
            tmem_wait_st();
            tc_fence_before();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&a_full[as]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&w_empty[s]);
      }
    }
  } else if (warp >= 12 && warp < 16) {
    // ---------------------------------------------------- epilogue ---
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    uint32_t di = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < n_units && ok; u += gridDim.x, ++di) {
      int e, mt, rb, nr, ws0, ws1, kc0, kc1;
      unit_range(u, e, mt, rb, nr, ws0, ws1, kc0, kc1);
      const int ds = di % DB;
      const int feat = mt * 128 + row;
      const int slot = __ldg(p.slot_table + e);
      const uint8_t* sbase = p.pool + size_t(slot) * size_t(p.slot_bytes);
      float gsc[NMAT];
#pragma unroll
      for (int m = 0; m < NMAT; ++m) gsc[m] = __ldg(reinterpret_cast<const float*>(sbase + p.global_off[m]));
      if (NMAT == 2) {   // G' and U' of the normalised rows (exact: a power of two)
#pragma unroll
        for (int m = 0; m < NMAT; ++m) gsc[m] *= kRowNormInv;
      }
      const bool split = p.splits > 1;
      // row factors of the unit's token rows, one coalesced load per 32 rows
      // issued before the accumulators are ready; lane j of group g holds
      // row 32 g + j and the block loop broadcasts them with shuffles
      constexpr int kGroups = (BN + 31) / 32;
      float tsl[kGroups];
#pragma unroll
      for (int g = 0; g < kGroups; ++g)
        tsl[g] = !split && g * 32 + lane < nr ? token_factor(p, rb + g * 32 + lane) : 1.0f;
      if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&d_full[ds], (di / DB) & 1, kTagDFull, di, u)))) break;
      tc_fence_after();
      const int n_eff = (nr + 15) & ~15;
      // 16-column blocks, the tensor-memory load of block b + 1 in flight while
      // block b is computed; the accumulator buffer is handed back as soon as
      // its last block has been loaded
      uint32_t v[2][NMAT][16];
      const uint32_t dcol = tmem + lane_base + ds * NMAT * BN;
      if (n_eff > 0) {
#pragma unroll
        for (int m = 0; m < NMAT; ++m) tmem_ld_32x32b_x16(dcol + m * BN, v[0][m]);
      }
      bool released = false;
      // Two versions of the block loop: rows whose factors are all 1 (every
      // row of activations of ordinary magnitude) skip the per-row factor --
      // a broadcast and two multiplies per element, which in the down GEMM's
      // epilogue are as long as the unit's MMAs.  The test is warp-uniform.
      bool unit_scaled = false;
#pragma unroll
      for (int g = 0; g < kGroups; ++g) unit_scaled |= tsl[g] != 1.0f;
      unit_scaled = __any_sync(0xFFFFFFFFu, unit_scaled);
      auto blocks = [&](auto scaled_tag) {
        constexpr bool kScaled = decltype(scaled_tag)::value;
#pragma unroll
        for (int bk = 0; bk < BN / 16; ++bk) {
          const int n0 = bk * 16;
          if (n0 >= n_eff) break;
          tmem_wait_ld();
          if (n0 + 16 < n_eff) {
#pragma unroll
            for (int m = 0; m < NMAT; ++m) tmem_ld_32x32b_x16(dcol + m * BN + n0 + 16, v[(bk + 1) & 1][m]);
          } else {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[ds]);
            released = true;
          }
          const uint32_t (&w)[NMAT][16] = v[bk & 1];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int n = n0 + i;
            const float ts = kScaled ? __shfl_sync(0xFFFFFFFFu, tsl[bk >> 1], (bk & 1) * 16 + i) : 1.0f;
            if (n >= nr) break;
            if (split) {
#pragma unroll
              for (int m = 0; m < NMAT; ++m)
                p.partials[(size_t(u) * NMAT + m) * 128 * BN + size_t(n) * 128 + row] = __uint_as_float(w[m][i]);
            } else if (feat < p.M) {
              float r;
              if (NMAT == 2) {
                r = kScaled ? silu_mul(gsc[0] * __uint_as_float(w[0][i]), gsc[NMAT - 1] * __uint_as_float(w[NMAT - 1][i]), ts)
                            : silu_mul1(gsc[0] * __uint_as_float(w[0][i]), gsc[NMAT - 1] * __uint_as_float(w[NMAT - 1][i]));
              } else {
                r = kScaled ? down_out(gsc[0], __uint_as_float(w[0][i]), ts) : gsc[0] * __uint_as_float(w[0][i]);
              }
              store_out<NMAT>(p.out, size_t(rb + n) * p.M + feat, r);
            }
          }
        }
      };
      if (unit_scaled) blocks(std::true_type{});
      else blocks(std::false_type{});
      if (!released) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&d_empty[ds]);
      }
      if (split) {
        // this warp's 32 rows: the last of the `splits` warps to arrive sums
        // the partials in split order and writes the result
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(p.counters + (u / p.splits) * 4 + quarter, 1) == p.splits - 1;
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (last) {
          __threadfence();
          const int u0 = u - (p.units[u].w >> 16);
          for (int n = 0; n < nr; ++n) {
            float acc[NMAT];
#pragma unroll
            for (int m = 0; m < NMAT; ++m) acc[m] = 0.0f;
            for (int sp = 0; sp < p.splits; ++sp) {
#pragma unroll
              for (int m = 0; m < NMAT; ++m)
                acc[m] += __ldcg(p.partials + (size_t(u0 + sp) * NMAT + m) * 128 * BN + size_t(n) * 128 + row);
            }
            if (feat < p.M) {
              float r;
              const float ts = token_factor(p, rb + n);
              if (NMAT == 2) {
                r = silu_mul(gsc[0] * acc[0], gsc[NMAT - 1] * acc[NMAT - 1], ts);
              } else {
                r = down_out(gsc[0], acc[0], ts);
              }
              store_out<NMAT>(p.out, size_t(rb + n) * p.M + feat, r);
            }
          }
          if (lane == 0) p.counters[(u / p.splits) * 4 + quarter] = 0;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  pdl_launch_dependents();   // the next kernel's CTAs may now take this SM's place
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ x to f16 ---

// ------------------------------------------------------ prep kernel ---
//
// One launch, two independent jobs that both need only the permutation:
//   blocks [0, nsched)   the two work lists and the counter resets
//   blocks [nsched, ..)  the f16 activations in permuted row order
struct PrepParams {
  // work lists
  const int32_t* offsets;
  const int32_t* slot_table;
  int E, num_slots, nsched;
  int bn1, mt1, s1, bn2, mt2, s2;
  int4* units1;
  int4* units2;
  int* counts;                 // [0] units of GEMM1, [1] of GEMM2, [3] decode unit queue
  int* counters1;
  int ncnt1;
  int* counters2;
  int ncnt2;
  int* tile_done;
  int ndone;
  // activations
  const uint4* x;
  const int32_t* perm_src;
  int P, k_top, H;
  uint4* x_perm;
  float* rowscale;
};

__device__ int block_exclusive_scan(int v, int* smem_warp_sums);

// Work lists.  Unit u = ((tile * m_tiles) + m_tile) * splits + split, tiles
// numbered in expert order, so the splits of one output tile are
// consecutive.  Every schedule block derives the experts' first tiles (each
// thread 4 experts, E <= 1024) and writes a strided share of the units, each
// unit's expert found by binary search over the first tiles.
__device__ void prep_schedule(const PrepParams& p, int b) {
  __shared__ int warp_sums[32];
  __shared__ int start1[kMaxExperts + 1], start2[kMaxExperts + 1];
  __shared__ int s_rb[kMaxExperts], s_n[kMaxExperts], s_slot[kMaxExperts];
  const int E = p.E;
  int c1[4], c2[4], sum1 = 0, sum2 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * threadIdx.x + i;
    int n = 0, rb = 0, slot = 0;
    if (e < E) {
      rb = p.offsets[e];
      n = p.offsets[e + 1] - rb;
      if (n > 0) {
        slot = p.slot_table[e];
        if (slot < 0) { if (b == 0) set_device_status(FT_DEV_NOT_RESIDENT); n = 0; }
        else if (slot >= p.num_slots) { if (b == 0) set_device_status(FT_DEV_BAD_INDEX); n = 0; }
      }
      s_rb[e] = rb;
      s_n[e] = n;
      s_slot[e] = slot;
    }
    c1[i] = (n + p.bn1 - 1) / p.bn1;
    c2[i] = (n + p.bn2 - 1) / p.bn2;
    sum1 += c1[i];
    sum2 += c2[i];
  }
  int ex1 = block_exclusive_scan(sum1, warp_sums);
  int ex2 = block_exclusive_scan(sum2, warp_sums);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = 4 * threadIdx.x + i;
    if (e < E) { start1[e] = ex1; start2[e] = ex2; }
    ex1 += c1[i];
    ex2 += c2[i];
  }
  if (threadIdx.x == blockDim.x - 1) { start1[E] = ex1; start2[E] = ex2; }   // the totals
  __syncthreads();
  const int stride = blockDim.x * p.nsched, first = threadIdx.x + blockDim.x * b;
  auto fill = [&](const int* start, int bn, int mt, int sp, int4* units) {
    const int total = start[E] * mt * sp;
    for (int u = first; u < total; u += stride) {
      const int tile = u / (mt * sp), rem = u - tile * (mt * sp);
      int lo = 0, hi = E;                 // last expert whose first tile is <= tile
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (start[mid] <= tile) lo = mid; else hi = mid;
      }
      const int t = tile - start[lo];
      units[u] = make_int4(lo | (s_slot[lo] << 10), rem / sp, s_rb[lo] + t * bn,
                           min(bn, s_n[lo] - t * bn) | ((rem % sp) << 16));
    }
    return total;
  };
  const int total1 = fill(start1, p.bn1, p.mt1, p.s1, p.units1);
  const int total2 = fill(start2, p.bn2, p.mt2, p.s2, p.units2);
  if (b == 0 && threadIdx.x == 0) {
    p.counts[0] = total1;
    p.counts[1] = total2;
    p.counts[2] = 0;
    p.counts[3] = 0;   // decode unit queue
  }
  for (int i = first; i < p.ncnt1; i += stride) p.counters1[i] = 0;
  for (int i = first; i < p.ncnt2; i += stride) p.counters2[i] = 0;
  for (int i = first; i < p.ndone; i += stride) p.tile_done[i] = 0;
}

__device__ __forceinline__ float bf16x2_absmax(uint32_t w) {
  return fmaxf(fabsf(__uint_as_float(w << 16)), fabsf(__uint_as_float(w & 0xFFFF0000u)));
}
// x * fa * fb to f16, eight values.  fa, fb are powers of two (two factors, so
// that a scaling by up to 2^147 needs no factor outside the fp32 range).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4& v, float fa, float fb) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w[q] << 16) * fa * fb,
                                        __uint_as_float(w[q] & 0xFFFF0000u) * fa * fb);
    o[q] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// The row exponent e_r of a row whose largest magnitude is m (finite):
// 0 when m is in [2, 8) (rows of ordinary magnitude keep the factor 1) or
// m = 0, else the e_r with m * 2^-e_r in [4, 8).
__device__ __forceinline__ int row_exp_of_max(float m) {
  if (m == 0.0f || (m >= 2.0f && m < 8.0f)) return 0;
  int e;
  frexpf(m, &e);                                 // m = f * 2^e, f in [0.5, 1); exact for subnormals too
  return e - 3;                                  // m * 2^-(e - 3) = 8 f in [4, 8)
}

// The row exponent from the row's largest magnitude (warp-wide max first); 0
// for a non-finite row, which also records FT_DEV_F16_RANGE.
__device__ __forceinline__ int prep_row_exp(float m) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  if (!(m <= 3.4028235e38f)) {
    set_device_status(FT_DEV_F16_RANGE);         // inf or nan input
    return 0;
  }
  return row_exp_of_max(m);
}

// One warp per permuted row r (token t = perm_src[r] / k): writes
// x_perm[r] = f16(x[t] * 2^(12 - e_r)) and rowscale[r] = 2^e_r, e_r the row
// exponent (so the converted row's largest magnitude is in [2^13, 2^15)).
// Every finite bf16 row qualifies (e_r in [-135, 125]).  The f16 conversion
// is exact for every element of the row within a factor 2^30 of the row's
// largest magnitude (bf16 has 8 significant bits; f16 represents those
// exactly down to 2^-17); smaller elements round, to f16 subnormals, with an
// absolute error of at most 2^-25 in converted units, below 2^-38 max|x[t]|.
// Rows in permuted order make each expert group's tokens one contiguous
// block, so the GEMM loads them as plain tiles.  Rows of up to 256 * kRegVec
// values are read once into registers with all loads in flight together (the
// kernel is latency-bound at decode sizes); longer rows are read twice.
template <int kRegVec>   // 16-byte vectors per lane kept in registers
__device__ void prep_rows(const PrepParams& p, int b) {
  const int lane = threadIdx.x & 31;
  const int r = b * (blockDim.x / 32) + threadIdx.x / 32;
  if (r >= p.P) return;
  const int t = __ldg(p.perm_src + r) / p.k_top;
  const int nv = p.H / 8;
  const uint4* row = p.x + size_t(t) * nv;
  uint4* out = p.x_perm + size_t(r) * nv;
  if (kRegVec > 0 && nv <= 32 * kRegVec) {
    uint4 v[kRegVec > 0 ? kRegVec : 1];
#pragma unroll
    for (int i = 0; i < kRegVec; ++i) {
      const int c = lane + 32 * i;
      v[i] = c < nv ? __ldg(row + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < kRegVec; ++i)
      m = fmaxf(m, fmaxf(fmaxf(bf16x2_absmax(v[i].x), bf16x2_absmax(v[i].y)),
                         fmaxf(bf16x2_absmax(v[i].z), bf16x2_absmax(v[i].w))));
    const int e = prep_row_exp(m);
    const int sx = 12 - e, sa = sx >> 1;
    const float fa = ldexpf(1.0f, sa), fb = ldexpf(1.0f, sx - sa);
    if (lane == 0) p.rowscale[r] = ldexpf(1.0f, e);
#pragma unroll
    for (int i = 0; i < kRegVec; ++i) {
      const int c = lane + 32 * i;
      if (c < nv) out[c] = bf16x8_to_f16x8(v[i], fa, fb);
    }
    return;
  }
  float m = 0.0f;
  for (int c = lane; c < nv; c += 32) {
    const uint4 v = __ldg(row + c);
    m = fmaxf(m, fmaxf(fmaxf(bf16x2_absmax(v.x), bf16x2_absmax(v.y)), fmaxf(bf16x2_absmax(v.z), bf16x2_absmax(v.w))));
  }
  const int e = prep_row_exp(m);
  const int sx = 12 - e, sa = sx >> 1;
  const float fa = ldexpf(1.0f, sa), fb = ldexpf(1.0f, sx - sa);
  if (lane == 0) p.rowscale[r] = ldexpf(1.0f, e);
  for (int c = lane; c < nv; c += 32) out[c] = bf16x8_to_f16x8(__ldg(row + c), fa, fb);
}

// Register budgets: rows held in registers (kRegVec 16-byte vectors a lane)
// take 2 CTAs an SM at 12 vectors, 3 at 8; rows read twice (kRegVec = 0)
// take 5.  More CTAs keep more of the permuted-row writes of prefill-sized
// batches in flight.
template <int kRegVec>
__global__ void __launch_bounds__(256, kRegVec == 0 ? 5 : kRegVec <= 8 ? 3 : 2) ffn_prep_kernel(const PrepParams p) {
  pdl_enter();
  if (int(blockIdx.x) < p.nsched) prep_schedule(p, blockIdx.x);
  else prep_rows<kRegVec>(p, blockIdx.x - p.nsched);
}

}  // namespace ftmoe
