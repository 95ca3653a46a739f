// Host side of the expert FFN: variant and split-K planning, workspace layout,
// TMA tensor maps, and the launches (schedule kernel, then the two grouped
// GEMMs of the chosen variant).
#include <cuda.h>
#include <cudaTypedefs.h>
#include "sm100.cuh"

namespace ftmoe {

// --------------------------------------------------------------- host ---

struct GemmShape { int bn, splits, sps, ws, bs, as, db; };

struct FfnPlan {
  bool decode;
  bool gu_smem;        // gate/up GEMM in the large-group shape (A in shared memory)
  bool small;          // both GEMMs in the small-group shape (64-row token tiles, four A slots)
  GemmShape g1, g2;
  int mt1, mt2, nkw1, nkw2, nkc1, nkc2;
  long long max_tiles1, max_tiles2;
  // workspace layout (byte offsets)
  size_t off_h, off_x16, off_rowscale, off_units1, off_units2, off_counts, off_cnt1, off_cnt2, off_done, off_part1,
      off_part2, total;
  long long max_units1, max_units2;
  int cnt_per;
};

static inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Split-K factor: a divisor of the K-stage count (all units of one launch do
// equal work) that minimises the makespan of the persistent grid, i.e.
// ceil(units * S / SMs) / (units * S / SMs), plus a charge per extra split for
// the partial sums it writes and reduces (`split_cost`, relative to one
// unit's own traffic).
static int choose_splits(double units_est, int nkw, int num_sms, double split_cost, int* sps_out) {
  int best = 1;
  double best_cost = 1e30;
  for (int s = 1; s <= std::min(nkw, 16); ++s) {
    if (nkw % s) continue;
    const double work = units_est * s / num_sms;   // waves of equal units
    const double cost = ceil(work - 1e-9) / work * (1.0 + split_cost * (s - 1));
    if (cost < best_cost - 1e-12) { best_cost = cost; best = s; }
  }
  *sps_out = nkw / best;
  return best;
}

// Prefill tile shapes <token rows (MMA N), weight stages, token stages, A
// stages, accumulator buffers, K per chunk, A in shared memory> of the two
// tcgen05 GEMMs.  Tensor memory holds DB * NMAT * BN accumulator columns plus,
// with A in tensor memory, AS * NMAT * KC / 2 for A.
//   gate/up, groups of up to a few hundred rows: A in tensor memory, 96-row
//     token tiles (the deeper weight ring keeps the weight stream going);
//   gate/up, large groups (mean >= kGateUpSmemRows rows per active expert):
//     A in shared memory, so that tensor memory holds two 128-column
//     accumulator buffers per matrix, with three A slots (measured on a B200:
//     wide_T8192 gate/up 1213 vs 1392 us, prefill_zipf_T4096 314 vs 330 us;
//     slots512_T8192 with 160 rows per expert 581 vs 525 us, so it keeps the
//     first shape).
constexpr int kPreBN1 = 96, kPreWS1 = 3, kPreBS1 = 4, kPreAS1 = 2, kPreDB1 = 2, kPreKC1 = 64, kPreAM1 = 0;
constexpr int kPreBN1S = 128, kPreWS1S = 2, kPreBS1S = 3, kPreAS1S = 3, kPreDB1S = 2, kPreKC1S = 64, kPreAM1S = 1;
constexpr double kGateUpSmemRows = 192.0;
// Token rows of up to 2048 values: converted from registers (8 vectors a lane)
// or read twice (0); see ffn_prep_kernel.
constexpr int kPrepVecSmallH = 8;
constexpr int kPreBN2 = 192, kPreWS2 = 3, kPreBS2 = 3, kPreAS2 = 2, kPreDB2 = 2, kPreKC2 = 128, kPreAM2 = 0;
//   both GEMMs, small groups (mean < kSmallGroupRows rows per active expert):
//     64-row token tiles, which leave tensor memory for four A slots (gate/up:
//     2 x 2 x 64 accumulator columns + 4 x 2 x 32; down: 2 x 64 + 4 x 64).
//     With a few dozen rows per group each chunk's MMAs are short, and the
//     A slot's round trip (dequantise -> MMA -> release) sets the pace; two
//     slots more keep twice as many chunks in flight.
constexpr int kPreBN1T = 64, kPreWS1T = 3, kPreBS1T = 4, kPreAS1T = 4, kPreDB1T = 2, kPreKC1T = 64, kPreAM1T = 0;
constexpr int kPreBN2T = 64, kPreWS2T = 3, kPreBS2T = 4, kPreAS2T = 4, kPreDB2T = 2, kPreKC2T = 128, kPreAM2T = 0;
constexpr double kSmallGroupRows = 48.0;
static_assert(kPreKC1T == kPreKC1 && kPreKC1S == kPreKC1 && kPreKC2T == kPreKC2, "one chunk size per GEMM");

// Decode split-K.  With at least as many units as SMs: none (the queue keeps
// every SM busy).  With fewer: the split that minimises the stages on the
// busiest CTA -- ceil(units * s / SMs) units of sps = ceil(nkw / s) stages --
// the fewest splits among equals.  A split need not divide the stage count:
// the last one takes what is left (never nothing, as s = ceil(nkw / sps)).
// At a few tokens the kernel is latency-bound, and each extra split's
// partial-sum exchange lengthens the chain from the first weight stage to
// the last output, so a second wave of units is worth it only where it
// shortens that chain.  (Measured on a B200: the 48-layer wide_decode_T1
// sweep 40.4 vs 41.0 us per layer, slots512_T1 33.9 vs 34.9 us, against the
// largest split count that divides the stages and keeps one wave.)
static int decode_splits(double units_est, int nkw, int num_sms, int* sps_out) {
  int best = 1, best_sps = nkw;
  if (units_est < num_sms) {
    double best_cost = 1e30;
    for (int sps = nkw; sps >= 1; --sps) {
      const int s = (nkw + sps - 1) / sps;
      if (s > 16) break;
      const double cost = ceil(units_est * s / num_sms - 1e-9) * sps;
      if (cost < best_cost - 1e-9) { best_cost = cost; best = s; best_sps = sps; }
    }
  }
  *sps_out = best_sps;
  return best;
}

// Variant choice: groups of a few token rows (mean rows per active expert
// <= kDecodeMeanRows) are bound by the weight bytes and take the
// weight-streaming decode kernel (both GEMMs in one launch, 16-row token
// units); larger groups take the tcgen05 kernel (128-row tiles, 128-row
// token units).
constexpr double kDecodeMeanRows = 16.0;

static FfnPlan plan_ffn(int T, int H, int I, int E, int k, int num_sms) {
  FfnPlan pl{};
  const long long P = (long long)T * k;
  const double distinct = E * (1.0 - pow(1.0 - double(k) / E, double(T)));
  const double mean_rows = distinct > 0 ? double(P) / distinct : 0.0;
  pl.decode = mean_rows <= kDecodeMeanRows;
  pl.mt1 = (I + (pl.decode ? kDecFeat1 : 128) - 1) / (pl.decode ? kDecFeat1 : 128);
  pl.mt2 = (H + (pl.decode ? kDecRows : 128) - 1) / (pl.decode ? kDecRows : 128);
  pl.nkw1 = (H + kKW - 1) / kKW;
  pl.nkw2 = (I + kKW - 1) / kKW;
  pl.nkc1 = (H + kPreKC1 - 1) / kPreKC1;
  pl.nkc2 = (I + kPreKC2 - 1) / kPreKC2;
  if (pl.decode) {
    pl.g1 = {kDecBN, 1, 0, 4, 0, 0, 0};
    pl.g2 = {kDecBN, 1, 0, 4, 0, 0, 0};
  } else {
    pl.gu_smem = mean_rows >= kGateUpSmemRows;
    pl.small = mean_rows < kSmallGroupRows;
    pl.g1 = pl.gu_smem ? GemmShape{kPreBN1S, 1, 0, kPreWS1S, kPreBS1S, kPreAS1S, kPreDB1S}
          : pl.small   ? GemmShape{kPreBN1T, 1, 0, kPreWS1T, kPreBS1T, kPreAS1T, kPreDB1T}
                       : GemmShape{kPreBN1, 1, 0, kPreWS1, kPreBS1, kPreAS1, kPreDB1};
    pl.g2 = pl.small ? GemmShape{kPreBN2T, 1, 0, kPreWS2T, kPreBS2T, kPreAS2T, kPreDB2T}
                     : GemmShape{kPreBN2, 1, 0, kPreWS2, kPreBS2, kPreAS2, kPreDB2};
  }
  const double tiles_per_expert1 = std::max(1.0, ceil(mean_rows / pl.g1.bn));
  const double tiles_per_expert2 = std::max(1.0, ceil(mean_rows / pl.g2.bn));
  const double est_tiles1 = std::max(1.0, ceil(distinct) * tiles_per_expert1);
  const double est_tiles2 = std::max(1.0, ceil(distinct) * tiles_per_expert2);
  if (pl.decode) {
    pl.g1.splits = decode_splits(est_tiles1 * pl.mt1, pl.nkw1, num_sms, &pl.g1.sps);
    pl.g2.splits = decode_splits(est_tiles2 * pl.mt2, pl.nkw2, num_sms, &pl.g2.sps);
  } else {
    // prefill partials are full 128 x 128 fp32 tiles: split only to fill the GPU
    const double split_cost1 = est_tiles1 * pl.mt1 >= num_sms ? 1.0 : 0.15;
    const double split_cost2 = est_tiles2 * pl.mt2 >= num_sms ? 1.0 : 0.15;
    pl.g1.splits = choose_splits(est_tiles1 * pl.mt1, pl.nkw1, num_sms, split_cost1, &pl.g1.sps);
    pl.g2.splits = choose_splits(est_tiles2 * pl.mt2, pl.nkw2, num_sms, split_cost2, &pl.g2.sps);
  }
  const long long active = std::min<long long>(E, P);
  pl.max_tiles1 = active + P / pl.g1.bn;
  pl.max_tiles2 = active + P / pl.g2.bn;
  pl.max_units1 = pl.max_tiles1 * pl.mt1 * pl.g1.splits;
  pl.max_units2 = pl.max_tiles2 * pl.mt2 * pl.g2.splits;
  // split-K counters per (tile, m-tile): one per epilogue warp of the kernel
  const int cnt_per = pl.decode ? 16 : 4;
  const size_t part_unit1 = pl.decode ? size_t(kDecPartialBytes) : size_t(2) * 128 * pl.g1.bn * 4;
  const size_t part_unit2 = pl.decode ? size_t(kDecPartialBytes) : size_t(1) * 128 * pl.g2.bn * 4;
  size_t o = 0;
  pl.off_h = o;       o = align256(o + size_t(P) * I * 2);
  pl.off_x16 = o;     o = align256(o + size_t(P) * H * 2);   // f16 activations, permuted rows
  pl.off_rowscale = o; o = align256(o + size_t(P) * 4);
  pl.off_units1 = o;  o = align256(o + size_t(pl.max_units1) * 16);
  pl.off_units2 = o;  o = align256(o + size_t(pl.max_units2) * 16);
  pl.off_counts = o;  o = align256(o + 16);   // [0] units of GEMM1, [1] of GEMM2, [2] any token prescaled, [3] queue
  pl.off_cnt1 = o;    o = align256(o + size_t(pl.max_tiles1 * pl.mt1) * cnt_per * 4);
  pl.off_cnt2 = o;    o = align256(o + size_t(pl.max_tiles2 * pl.mt2) * cnt_per * 4);
  pl.off_done = o;    o = align256(o + size_t(pl.max_tiles1) * 4);   // decode: h published per token tile
  pl.off_part1 = o;
  if (pl.g1.splits > 1) o = align256(o + size_t(pl.max_units1) * part_unit1);
  pl.off_part2 = o;
  if (pl.g2.splits > 1) o = align256(o + size_t(pl.max_units2) * part_unit2);
  pl.total = o;
  pl.cnt_per = cnt_per;
  return pl;
}

static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// codes: [rows, K/2] bytes per slot, 128 x 128-byte boxes, 128-byte swizzle.
// scales: [rows, ld_scale] bytes per slot, 128 x 16-byte boxes.
// Stage-tiled slots: codes [S][rows][128] and scales [S][rows][16] per slot,
// 4-D maps (bytes, rows, stage, slot) with the same boxes, so that a box is
// one contiguous block of memory.
static bool make_weight_maps(const uint8_t* pool, const ft_nvfp4_slot_layout& L, int mat, int rows, int K,
                             int box_rows, CUtensorMap* codes, CUtensorMap* scales) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  if (L.tiled) {
    const cuuint64_t stages = cuuint64_t((K + 255) / 256);
    const cuuint32_t es4[4] = {1, 1, 1, 1};
    {
      const cuuint64_t dims[4] = {128, cuuint64_t(rows), stages, cuuint64_t(L.num_slots)};
      const cuuint64_t strides[3] = {128, cuuint64_t(rows) * 128, cuuint64_t(L.slot_bytes)};
      const cuuint32_t box[4] = {128, cuuint32_t(box_rows), 1, 1};
      if (enc(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, (void*)(pool + L.codes_off[mat]), dims, strides, box, es4,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    }
    {
      const cuuint64_t dims[4] = {16, cuuint64_t(rows), stages, cuuint64_t(L.num_slots)};
      const cuuint64_t strides[3] = {16, cuuint64_t(rows) * 16, cuuint64_t(L.slot_bytes)};
      const cuuint32_t box[4] = {16, cuuint32_t(box_rows), 1, 1};
      if (enc(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, (void*)(pool + L.scales_off[mat]), dims, strides, box, es4,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    }
    return true;
  }
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  {
    const cuuint64_t dims[3] = {cuuint64_t(K / 2), cuuint64_t(rows), cuuint64_t(L.num_slots)};
    const cuuint64_t strides[2] = {cuuint64_t(K / 2), cuuint64_t(L.slot_bytes)};
    const cuuint32_t box[3] = {128, cuuint32_t(box_rows), 1};
    if (enc(codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void*)(pool + L.codes_off[mat]), dims, strides, box,
            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  {
    const cuuint64_t dims[3] = {cuuint64_t(L.ld_scale[mat]), cuuint64_t(rows), cuuint64_t(L.num_slots)};
    const cuuint64_t strides[2] = {cuuint64_t(L.ld_scale[mat]), cuuint64_t(L.slot_bytes)};
    const cuuint32_t box[3] = {16, cuuint32_t(box_rows), 1};
    if (enc(scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void*)(pool + L.scales_off[mat]), dims, strides, box,
            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// Activation rows (bf16 [rows, K]) as the MMA's B operand, 64-column (128-byte)
// boxes with the 128-byte swizzle: box_rows contiguous rows (the decode
// kernel's token tile, or a prefill GEMM's whole BN-row token tile).
static bool make_act_map(const void* base, int rows, int K, int box_rows, CUtensorMap* m) {  // f16 rows
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {cuuint64_t(K), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(K) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  const cuuint32_t elem_strides[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NMAT, int BN, int WS, int BS, int AS, int DB, int KC, int FMT, int AM>
static cudaError_t launch_gemm(const FfnParams& p, int grid, const CUtensorMap& c0, const CUtensorMap& s0,
                               const CUtensorMap& c1, const CUtensorMap& s1, const CUtensorMap& act,
                               cudaStream_t s) {
  ProfileScope prof(NMAT == 2 ? FT_KERNEL_GEMM_GATE_UP : FT_KERNEL_GEMM_DOWN, s);
  using Cfg = FfnCfg<NMAT, BN, WS, BS, AS, DB, KC, AM>;
  auto kern = ffn_gemm_kernel<NMAT, BN, WS, BS, AS, DB, KC, FMT, AM>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(kern, dim3(grid), dim3(kThreads), Cfg::kSmemBytes, s, p, c0, s0, c1, s1, act);
}

static int device_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

static cudaError_t launch_ffn(const void* x, int T, int H, int I, int E, int k, const int32_t* perm_src,
                              const int32_t* offsets, const int32_t* slot_table, const void* pool_v,
                              const ft_nvfp4_slot_layout& L, void* out_perm, void* ws, cudaStream_t s,
                              const char** why) {
  const int num_sms = device_sm_count();
  const FfnPlan pl = plan_ffn(T, H, I, E, k, num_sms);
  const uint8_t* pool = static_cast<const uint8_t*>(pool_v);
  uint8_t* w = static_cast<uint8_t*>(ws);
  CUtensorMap tmc[3], tms[3];
  const int rows[3] = {I, I, H}, Ks[3] = {H, H, I};
  for (int m = 0; m < 3; ++m)
    if (!make_weight_maps(pool, L, m, rows[m], Ks[m], 128, &tmc[m], &tms[m])) {
      *why = "cuTensorMapEncodeTiled failed for the slot pool";
      return cudaErrorInvalidValue;
    }
  int4* units1 = reinterpret_cast<int4*>(w + pl.off_units1);
  int4* units2 = reinterpret_cast<int4*>(w + pl.off_units2);
  int* counts = reinterpret_cast<int*>(w + pl.off_counts);
  int* cnt1 = reinterpret_cast<int*>(w + pl.off_cnt1);
  int* cnt2 = reinterpret_cast<int*>(w + pl.off_cnt2);
  __half* h = reinterpret_cast<__half*>(w + pl.off_h);
  __half* x16 = reinterpret_cast<__half*>(w + pl.off_x16);
  float* rowscale = reinterpret_cast<float*>(w + pl.off_rowscale);
  cudaError_t err;
  {
    PrepParams pp{};
    pp.offsets = offsets;
    pp.slot_table = slot_table;
    pp.E = E;
    pp.num_slots = L.num_slots;
    pp.nsched = int(std::min<long long>(32, std::max<long long>(1, (pl.max_units1 + pl.max_units2) / 4096)));
    pp.bn1 = pl.g1.bn; pp.mt1 = pl.mt1; pp.s1 = pl.g1.splits;
    pp.bn2 = pl.g2.bn; pp.mt2 = pl.mt2; pp.s2 = pl.g2.splits;
    pp.units1 = units1;
    pp.units2 = units2;
    pp.counts = counts;
    pp.counters1 = cnt1;
    pp.ncnt1 = int(pl.max_tiles1 * pl.mt1 * pl.cnt_per);
    pp.counters2 = cnt2;
    pp.ncnt2 = int(pl.max_tiles2 * pl.mt2 * pl.cnt_per);
    pp.tile_done = reinterpret_cast<int*>(w + pl.off_done);
    pp.ndone = pl.decode ? int(pl.max_tiles1) : 0;
    pp.x = static_cast<const uint4*>(x);
    pp.perm_src = perm_src;
    pp.P = T * k;
    pp.k_top = k;
    pp.H = H;
    pp.x_perm = reinterpret_cast<uint4*>(x16);
    pp.rowscale = rowscale;
    ProfileScope prof(FT_KERNEL_PREP, s);
    err = launch_pdl(H <= 2048 ? ffn_prep_kernel<kPrepVecSmallH> : ffn_prep_kernel<12>,
                     dim3(pp.nsched + (T * k + 7) / 8), dim3(256), 0, s, pp);
  }
  if (err != cudaSuccess) return err;

  CUtensorMap tm_x, tm_h;
  if (!make_act_map(x16, T * k, H, pl.decode ? kDecBN : pl.g1.bn, &tm_x) ||
      !make_act_map(h, T * k, I, pl.decode ? kDecBN : pl.g2.bn, &tm_h)) {
    *why = "cuTensorMapEncodeTiled failed for the activations";
    return cudaErrorInvalidValue;
  }
  FfnParams p1{};
  p1.rowscale = rowscale;
  p1.perm_src = perm_src;
  p1.k_top = k;
  p1.K = H;
  p1.M = I;
  p1.nkw = pl.nkw1;
  p1.nkc = pl.nkc1;
  p1.splits = pl.g1.splits;
  p1.stages_per_split = pl.g1.sps;
  p1.units = units1;
  p1.num_units = counts;
  p1.slot_table = slot_table;
  p1.pool = pool;
  p1.slot_bytes = L.slot_bytes;
  p1.global_off[0] = L.global_off[FT_GATE];
  p1.global_off[1] = L.global_off[FT_UP];
  p1.out = h;
  p1.partials = reinterpret_cast<float*>(w + pl.off_part1);
  p1.counters = cnt1;
  p1.tiled = L.tiled;
  const int grid1 = int(std::min<long long>(num_sms, pl.max_units1));

  FfnParams p2 = p1;
  p2.perm_src = nullptr;
  p2.rowscale = rowscale;   // the same permuted rows: GEMM2 undoes the rows' normalisation of h
  p2.K = I;
  p2.M = H;
  p2.nkw = pl.nkw2;
  p2.nkc = pl.nkc2;
  p2.splits = pl.g2.splits;
  p2.stages_per_split = pl.g2.sps;
  p2.units = units2;
  p2.num_units = counts + 1;
  p2.global_off[0] = L.global_off[FT_DOWN];
  p2.global_off[1] = L.global_off[FT_DOWN];
  p2.out = out_perm;
  p2.partials = reinterpret_cast<float*>(w + pl.off_part2);
  p2.counters = cnt2;
  const int grid2 = int(std::min<long long>(num_sms, pl.max_units2));

  if (pl.decode) {
    DecodeParams dp{};
    dp.g[0] = p1;
    dp.g[1] = p2;
    dp.queue = counts + 3;
    dp.tile_done = reinterpret_cast<int*>(w + pl.off_done);
    dp.mt1 = pl.mt1;
    dp.mt2 = pl.mt2;
    const int grid = int(std::min<long long>(num_sms, pl.max_units1 + pl.max_units2));
    err = L.scale_format == FT_SCALE_MXFP4 ? launch_decode<FT_SCALE_MXFP4>(dp, grid, tmc, tms, tm_x, tm_h, s)
                                           : launch_decode<FT_SCALE_NVFP4>(dp, grid, tmc, tms, tm_x, tm_h, s);
  } else {
    const bool mx = L.scale_format == FT_SCALE_MXFP4;
    if (pl.gu_smem)
      err = mx ? launch_gemm<2, kPreBN1S, kPreWS1S, kPreBS1S, kPreAS1S, kPreDB1S, kPreKC1S, FT_SCALE_MXFP4, kPreAM1S>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s)
               : launch_gemm<2, kPreBN1S, kPreWS1S, kPreBS1S, kPreAS1S, kPreDB1S, kPreKC1S, FT_SCALE_NVFP4, kPreAM1S>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s);
    else if (pl.small)
      err = mx ? launch_gemm<2, kPreBN1T, kPreWS1T, kPreBS1T, kPreAS1T, kPreDB1T, kPreKC1T, FT_SCALE_MXFP4, kPreAM1T>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s)
               : launch_gemm<2, kPreBN1T, kPreWS1T, kPreBS1T, kPreAS1T, kPreDB1T, kPreKC1T, FT_SCALE_NVFP4, kPreAM1T>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s);
    else
      err = mx ? launch_gemm<2, kPreBN1, kPreWS1, kPreBS1, kPreAS1, kPreDB1, kPreKC1, FT_SCALE_MXFP4, kPreAM1>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s)
               : launch_gemm<2, kPreBN1, kPreWS1, kPreBS1, kPreAS1, kPreDB1, kPreKC1, FT_SCALE_NVFP4, kPreAM1>(p1, grid1, tmc[0], tms[0], tmc[1], tms[1], tm_x, s);
    if (err == cudaSuccess && pl.small)
      err = mx ? launch_gemm<1, kPreBN2T, kPreWS2T, kPreBS2T, kPreAS2T, kPreDB2T, kPreKC2T, FT_SCALE_MXFP4, kPreAM2T>(p2, grid2, tmc[2], tms[2], tmc[2], tms[2], tm_h, s)
               : launch_gemm<1, kPreBN2T, kPreWS2T, kPreBS2T, kPreAS2T, kPreDB2T, kPreKC2T, FT_SCALE_NVFP4, kPreAM2T>(p2, grid2, tmc[2], tms[2], tmc[2], tms[2], tm_h, s);
    else if (err == cudaSuccess)
      err = mx ? launch_gemm<1, kPreBN2, kPreWS2, kPreBS2, kPreAS2, kPreDB2, kPreKC2, FT_SCALE_MXFP4, kPreAM2>(p2, grid2, tmc[2], tms[2], tmc[2], tms[2], tm_h, s)
               : launch_gemm<1, kPreBN2, kPreWS2, kPreBS2, kPreAS2, kPreDB2, kPreKC2, FT_SCALE_NVFP4, kPreAM2>(p2, grid2, tmc[2], tms[2], tmc[2], tms[2], tm_h, s);
  }
  return err;
}

}  // namespace ftmoe
