// The whole MoE layer for decode-sized batches in ONE persistent launch:
// route -> permute -> gate/up GEMM + SwiGLU -> down GEMM -> combine.
//
// At a few tokens per expert the layer streams the weights of the experts it
// routes to, and what surrounds that stream -- four more launches, each a few
// microseconds of launch and dependency latency with almost no work -- costs
// as much as the stream itself at T = 1.  Here one grid (one CTA per SM) does
// every step:
//
//   phase 1  2T work items are claimed from a counter by whichever CTAs are
//            resident: routing token t (warp 0; the per-token code of
//            ft_moe_route, so the same ids and weight bits), and converting
//            row t to f16 with its power-of-two factor (the whole CTA; the
//            arithmetic of the separate path's prep kernel) into a
//            token-ordered f16 copy in the workspace.  Each finished item adds
//            one to a global count of routed tokens or of converted rows
//            (release), so routing and conversion run on different CTAs at
//            once and no wait depends on a CTA that has not started.
//   phase 2  every CTA waits (bounded) until all T tokens are routed, reads
//            the ids and builds, in its own shared memory, the expert counts,
//            offsets and token-tile tables: the unit list, with no further
//            grid-wide step.  Its weight producer starts streaming then, while
//            the other warps sort the pairs by expert (the counting sort of
//            ft_moe_permute: ascending pair index inside a group), wait until
//            all rows are converted and load the row factors; CTA 0 writes the
//            offsets and both permutation arrays out.
//   phase 3  the decode kernel's persistent unit queue (decode.cu): gate/up
//            units, then down units, 16-row token tiles, the same split-K
//            choice and the same summation order, so the expert outputs are
//            bit-identical to ft_moe_ffn_nvfp4's.  The token rows of a gate/up
//            unit are gathered from the token-ordered f16 copy by cp.async
//            (row r of the tile is token perm_src[r] / k) instead of a TMA box
//            of a permuted copy; down units read h by TMA as before.
//   phase 4  combine: each CTA publishes how many down units it finished
//            (one release after its last unit); once the count reaches the
//            number of down units, every CTA sums a strided share of the
//            output vectors in the order j = 0 .. k-1 with the combine
//            kernel's arithmetic, so y is bit-identical to ft_moe_combine's.
//
// Workspace counters (routed tokens, converted rows, the unit queue, down
// units done, CTAs done, h published per token tile, split-K arrivals) start at zero: the
// caller zero-fills the workspace once, and every call leaves them at zero
// again (each counter is reset by the last thread to use it; the last CTA to
// finish resets the rest, and everything after a call that recorded a device
// status).
#include <cuda.h>
#include <cuda_fp16.h>
#include "sm100.cuh"

namespace ftmoe {

constexpr int kLayerMaxT = 128;     // tokens
constexpr int kLayerMaxP = 1024;    // routed pairs (T * k)
constexpr int kLayerMaxE = 512;     // experts
constexpr int kLayerMiscInts = 48;
constexpr int kLayerTablesBytes = 4 * (4 * kLayerMaxP + kLayerMaxT + 4 * (kLayerMaxE + 1) + kLayerMiscInts);
constexpr int kLayerSmemBytes = kDecSmemBytes + kLayerTablesBytes;
static_assert(kLayerSmemBytes <= 227 * 1024, "shared memory budget");

// Barrier tags of the waits for every token to be routed / every row converted.
constexpr int kTagRouted = 11;
constexpr int kTagConverted = 12;
constexpr int kTagCombine = 13;    // the wait for every down unit before the combine
constexpr int kLayerCtrl = 6;      // control counters in the workspace

struct LayerParams {
  DecodeParams d;              // the FFN steps; d.g[*].units are unused (units come from the sort)
  const float* logits;         // [T, E]
  const uint4* x;              // [T, H] bf16
  int T, E, k, H, mode, npl, num_slots;
  int32_t* ids;                // [T, k] (out)
  float* wts;                  // [T, k] (out)
  int32_t* offsets;            // [E + 1] (out)
  int32_t* perm_src;           // [P] (out)
  int32_t* pair_to_row;        // [P] (out)
  float* y;                    // [T, H] (out)
  uint4* x16;                  // [T, H] f16, token order (workspace)
  float* rowscale;             // [T] row factors 2^e_t (workspace)
  int* ctrl;                   // [0] tokens routed, [1] unit queue, [2] CTAs done, [3] phase-1 items claimed,
                               // [4] rows converted, [5] down units done (workspace)
  int* tile_done;              // per token tile: h rows published (workspace)
  int* cnt1;                   // split-K arrivals of gate/up, n_cnt1 ints
  int* cnt2;                   // split-K arrivals of down, n_cnt2 ints
  int n_cnt1, n_cnt2, n_done;  // sizes of the counter arrays (for the reset after an error)
};

// Shared-memory tables built in phase 2.
struct LayerTables {
  int* ids;       // [P] expert of pair p (phase 2 scratch)
  int* ps;        // [P] row -> pair
  int* p2r;       // [P] pair -> row
  float* w;       // [P] routing weight of pair p
  float* rs;      // [T] row factor of token t
  int* off;       // [E + 1] group offsets
  int* start;     // [E + 1] first token tile of each expert (16-row tiles)
  int* slot;      // [E] slot of each expert (first the raw slot table)
  int* cur;       // [E] the scatter's cursors
  int* misc;      // [0] gate/up units, [1] all units, [2] abort / last CTA, [3] tiles,
                  // [4, 36) reduction scratch, [kMiscClaim] the claimed item,
                  // [kMiscConv] the wait for converted rows gave up
};
constexpr int kMiscClaim = 36;
constexpr int kMiscConv = 37;      // a wait of phase 2b or 4 gave up
constexpr int kMiscDown = 38;      // down units this CTA finished
// Named barrier of the warps that run phase 2b (all but the weight producer).
constexpr int kBarPhase2 = 1;

__device__ __forceinline__ LayerTables layer_tables(uint8_t* base) {
  LayerTables t;
  int* p = reinterpret_cast<int*>(base);
  t.ids = p;        p += kLayerMaxP;
  t.ps = p;         p += kLayerMaxP;
  t.p2r = p;        p += kLayerMaxP;
  t.w = reinterpret_cast<float*>(p); p += kLayerMaxP;
  t.rs = reinterpret_cast<float*>(p); p += kLayerMaxT;
  t.off = p;        p += kLayerMaxE + 1;
  t.start = p;      p += kLayerMaxE + 1;
  t.slot = p;       p += kLayerMaxE + 1;
  t.cur = p;        p += kLayerMaxE + 1;
  t.misc = p;
  return t;
}

// The descriptor of queue position q, in the format of the separate path's
// unit lists ({expert | slot << 10, m-tile, first row, rows | split << 16}),
// from the shared-memory tables.  Unit u of a GEMM is
// ((tile * m_tiles) + m_tile) * splits + split, tiles numbered in expert order.
__device__ __forceinline__ int4 layer_unit_desc(const LayerParams& p, const LayerTables& tb, int q, int n1, int E) {
  const int gemm = q < n1 ? 0 : 1;
  const int u = gemm ? q - n1 : q;
  const int mt_count = gemm ? p.d.mt2 : p.d.mt1;
  const int sp = p.d.g[gemm].splits;
  const int tile = u / (mt_count * sp), rem = u - tile * (mt_count * sp);
  int lo = 0, hi = E;                 // last expert whose first tile is <= tile
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (tb.start[mid] <= tile) lo = mid; else hi = mid;
  }
  const int t = tile - tb.start[lo];
  const int n = tb.off[lo + 1] - tb.off[lo];
  return make_int4(lo | (tb.slot[lo] << 10), rem / sp, tb.off[lo] + t * kDecBN,
                   min(kDecBN, n - t * kDecBN) | ((rem % sp) << 16));
}

__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Largest value over the block (every thread calls it); scratch: 32 floats.
__device__ float block_max(float v, float* scratch) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float m = lane < nw ? scratch[lane] : 0.0f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    if (lane == 0) scratch[0] = m;
  }
  __syncthreads();
  const float r = scratch[0];
  __syncthreads();
  return r;
}

// Phase 1, routing item: the top-k and weights of token t (warp 0 only).
__device__ void layer_route_token(const LayerParams& p, int t) {
  const int lane = threadIdx.x & 31;
  const float* row = p.logits + size_t(t) * p.E;
  int sel = 0;
  float w = 0.0f;
  switch (p.npl) {
    case 1: route_token<1>(row, p.E, p.k, p.mode, lane, sel, w); break;
    case 2: route_token<2>(row, p.E, p.k, p.mode, lane, sel, w); break;
    case 4: route_token<4>(row, p.E, p.k, p.mode, lane, sel, w); break;
    case 8: route_token<8>(row, p.E, p.k, p.mode, lane, sel, w); break;
    default: route_token<16>(row, p.E, p.k, p.mode, lane, sel, w); break;
  }
  if (lane < p.k) {
    p.ids[size_t(t) * p.k + lane] = sel;
    p.wts[size_t(t) * p.k + lane] = w;
  }
}

// Phase 1, conversion item: token t's row to f16 with its power-of-two factor
// (the prep kernel's arithmetic), and the factor (whole CTA).
__device__ void layer_convert_row(const LayerParams& p, int t, float* scratch) {
  const int nv = p.H / 8;
  const uint4* xr = p.x + size_t(t) * nv;
  float m = 0.0f;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) {
    const uint4 v = __ldg(xr + c);
    m = fmaxf(m, fmaxf(fmaxf(bf16x2_absmax(v.x), bf16x2_absmax(v.y)), fmaxf(bf16x2_absmax(v.z), bf16x2_absmax(v.w))));
  }
  m = block_max(m, scratch);
  int e = 0;
  if (!(m <= 3.4028235e38f)) {
    if (threadIdx.x == 0) set_device_status(FT_DEV_F16_RANGE);
  } else {
    e = row_exp_of_max(m);
  }
  const int sx = 12 - e, sa = sx >> 1;
  const float fa = ldexpf(1.0f, sa), fb = ldexpf(1.0f, sx - sa);
  uint4* out = p.x16 + size_t(t) * nv;
  for (int c = threadIdx.x; c < nv; c += blockDim.x) out[c] = bf16x8_to_f16x8(__ldg(xr + c), fa, fb);
  if (threadIdx.x == 0) p.rowscale[t] = ldexpf(1.0f, e);
}

// Bounded wait (one thread) until counter >= target; false (status recorded)
// if it gave up.
__device__ bool layer_wait_count(const int* counter, int target, int tag) {
  if (ld_acquire_gpu(counter) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t n = 0;
  while (ld_acquire_gpu(counter) < target) {
    __nanosleep(64);
    if ((++n & 15u) == 0 && globaltimer_ns() - t0 > 1000000000ull) {
      set_device_status_detail(FT_DEV_WAIT_TIMEOUT, tag, ld_acquire_gpu(counter), target,
                               (long long)((globaltimer_ns() - t0) / 1000));
      return false;
    }
  }
  return true;
}

// Phase 2a (whole CTA): once every token is routed, the expert counts,
// offsets and token-tile tables -- what the weight producer needs to start.
// tb.slot holds the raw slot table (loaded at kernel start).  Returns false if
// the wait for the routed tokens gave up.
__device__ bool layer_counts(const LayerParams& p, const LayerTables& tb, int* scan_scratch) {
  const int T = p.T, k = p.k, E = p.E, P = T * k;
  if (threadIdx.x == 0) tb.misc[2] = layer_wait_count(p.ctrl, T, kTagRouted) ? 0 : 1;
  __syncthreads();
  if (tb.misc[2]) return false;
  // everything phase 1 wrote is read through L2 (written during this kernel)
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    int e = __ldcg(p.ids + i);
    if (!valid_expert(e, E)) { set_device_status(FT_DEV_BAD_INDEX); e = -1; }
    tb.ids[i] = e;
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) tb.start[e] = 0;   // counts first
  __syncthreads();
  for (int i = threadIdx.x; i < P; i += blockDim.x)
    if (tb.ids[i] >= 0) atomicAdd(&tb.start[tb.ids[i]], 1);
  __syncthreads();
  // offsets: exclusive scan of the counts (E <= blockDim.x: one expert per thread)
  const int e = threadIdx.x;
  const int c = e < E ? tb.start[e] : 0;
  const int ex = block_exclusive_scan(c, scan_scratch);
  if (e < E) tb.off[e] = ex;
  if (e == E - 1) tb.off[E] = ex + c;
  // token tiles per expert (experts without rows, or not resident, have none)
  int tiles = 0, slot = 0;
  if (e < E && c > 0) {
    slot = tb.slot[e];
    if (slot < 0) { if (blockIdx.x == 0) set_device_status(FT_DEV_NOT_RESIDENT); }
    else if (slot >= p.num_slots) { if (blockIdx.x == 0) set_device_status(FT_DEV_BAD_INDEX); }
    else tiles = (c + kDecBN - 1) / kDecBN;
  }
  const int ts = block_exclusive_scan(tiles, scan_scratch);   // (synchronises the block)
  if (e < E) { tb.start[e] = ts; tb.cur[e] = ex; tb.slot[e] = tiles > 0 ? slot : 0; }
  if (e == E - 1) {
    tb.start[E] = ts + tiles;
    tb.misc[3] = ts + tiles;
    tb.misc[0] = (ts + tiles) * p.d.mt1 * p.d.g[0].splits;
    tb.misc[1] = tb.misc[0] + (ts + tiles) * p.d.mt2 * p.d.g[1].splits;
  }
  __syncthreads();
  return true;
}

// Phase 2b (every warp but the weight producer, nthreads of them): the
// scatter into the shared-memory permutation (ascending pair index inside a
// group), the routing weights, CTA 0's copies of the offsets and both
// permutations, and -- once every row is converted -- the row factors.
// Returns false if the wait for the converted rows gave up.
__device__ bool layer_scatter(const LayerParams& p, const LayerTables& tb, int nthreads, int tid) {
  const int T = p.T, k = p.k, E = p.E, P = T * k;
  for (int i = tid; i < P; i += nthreads) tb.w[i] = __ldcg(p.wts + i);
  if (tid < 32) scatter_chunk_warp<true>(tb.ids, 0, P, E, tb.cur, tb.ps, tb.p2r, P);
  if (tid == 32) tb.misc[kMiscConv] = layer_wait_count(p.ctrl + 4, T, kTagConverted) ? 0 : 1;
  named_bar_sync(kBarPhase2, nthreads);
  if (tb.misc[kMiscConv]) return false;
  for (int t = tid; t < T; t += nthreads) tb.rs[t] = __ldcg(p.rowscale + t);
  if (blockIdx.x == 0) {
    for (int i = tid; i <= E; i += nthreads) p.offsets[i] = tb.off[i];
    for (int i = tid; i < P; i += nthreads) {
      p.perm_src[i] = tb.ps[i];
      p.pair_to_row[i] = tb.p2r[i];
    }
  }
  named_bar_sync(kBarPhase2, nthreads);
  return true;
}

// The token rows of a gate/up unit, as one lane of the token loader sees
// them.  One 256-K stage is 512 chunks of 16 bytes (4 boxes of 64 K x 16 rows,
// 128-byte swizzle); lane l issues chunks c = l + 32 i, i = 0..15, which are
// box i / 4, row (l / 8) + 4 (i % 4) and 16-byte column l % 8 -- so a lane
// touches four rows, whose source rows and destination offsets it works out
// once per unit.
struct GatherRows {
  const uint4* src[4];   // the token's f16 row (token order), or null past the group
  uint32_t dst[4];       // byte offset of the chunk in its box
};

__device__ __forceinline__ GatherRows layer_gather_rows(const LayerParams& p, const LayerTables& tb, int rb, int nr,
                                                        int lane) {
  GatherRows g;
  const int nv = p.H / 8, j = lane & 7;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int row = (lane >> 3) + 4 * q;
    g.src[q] = row < nr ? p.x16 + size_t(tb.ps[rb + row] / p.k) * nv + j : nullptr;
    g.dst[q] = uint32_t(row * 128 + ((j ^ (row & 7)) << 4));
  }
  return g;
}

// One 256-K stage of those rows into the token boxes at bst; rows past the
// group and K past H are zero-filled.  Each lane then arrives on `bar` when
// its copies have landed.
__device__ __forceinline__ void layer_gather_stage(const LayerParams& p, const GatherRows& g, uint8_t* bst,
                                                   uint64_t* bar, int ws, int lane) {
  const int nv = p.H / 8;
  const int kv0 = ws * (kDecStageK / 8) + (lane & 7);
  const uint32_t b = smem_u32(bst);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int q = i & 3, bx = i >> 2;
    const int kv = kv0 + bx * 8;
    const bool live = g.src[q] != nullptr && kv < nv;
    cp_async_16(b + bx * kDecBBoxBytes + g.dst[q], live ? g.src[q] + (kv - (lane & 7)) : p.x16, live ? 16u : 0u);
  }
  cp_async_mbar_arrive_noinc(bar);
}

// Compute warp w's part of one unit: the decode kernel's dec_unit with the
// row factors from the shared-memory tables.
template <int NT, int FMT>
__device__ bool layer_unit(const LayerParams& p, const LayerTables& tb, const DecUnit& d, uint8_t* smem,
                           uint64_t* full, uint64_t* empty, const Abort& ab, uint64_t* unit_free,
                           const int4* unit_ent, uint64_t* hpub, int* hcount, int gu, uint32_t& si, int q, int w,
                           int lane) {
  const DecodeParams& dp = p.d;
  const int g = lane >> 2, t = lane & 3;
  const int r_lo = dec_row_lo(d.gemm, w, g), r_hi = dec_row_hi(d.gemm, w, g);
  int blo = 0, bhi = 0;
  if (FMT == FT_SCALE_MXFP4) {
    const FfnParams& G = dp.g[d.gemm];
    const uint8_t* sbase = G.pool + size_t(d.slot) * size_t(G.slot_bytes);
    blo = mx_bias(__ldg(reinterpret_cast<const float*>(sbase + G.global_off[0])));
    bhi = mx_bias(__ldg(reinterpret_cast<const float*>(sbase + G.global_off[1])));
  }
  float ts[NT][2];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int r = 8 * n + 2 * t + e;
      ts[n][e] = r < d.nr ? tb.rs[tb.ps[d.rb + r] / p.k] : 1.0f;
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
  DecConsts c;
  {
    const int4 ce = *unit_ent;
    c.g0 = __int_as_float(ce.y); c.g1 = __int_as_float(ce.z);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(unit_free);
  const bool fin = dec_epilogue<NT>(dp, d, c, w, lane, acc, ts);
  if (d.gemm == 0) {
    __syncwarp();
    if (fin && lane == 0) atomicAdd(&hcount[gu & 1], 1);
    mbar_arrive(&hpub[gu & 1]);
    return true;
  }
  (void)fin;
  return true;
}

template <int FMT>
__global__ void __launch_bounds__(kDecThreads, 1)
layer_decode_kernel(const LayerParams p, const __grid_constant__ CUtensorMap tm_c0,
                    const __grid_constant__ CUtensorMap tm_s0, const __grid_constant__ CUtensorMap tm_c1,
                    const __grid_constant__ CUtensorMap tm_s1, const __grid_constant__ CUtensorMap tm_c2,
                    const __grid_constant__ CUtensorMap tm_s2, const __grid_constant__ CUtensorMap tm_h) {
  pdl_enter();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDecStages * kDecStageBytes);
  uint64_t* empty = full + kDecStages;
  uint64_t* ufull = empty + kDecStages;
  uint64_t* uempty = ufull + kDecUnitRing;
  uint64_t* hpub = uempty + kDecUnitRing;
  int4* uent = reinterpret_cast<int4*>(hpub + 2);
  int4* udesc = uent + kDecUnitRing;
  int* hcount = reinterpret_cast<int*>(udesc + kDecUnitRing);
  int* abort_flag = hcount + 2;
  const LayerTables tb = layer_tables(smem_raw + kDecSmemBytes);   // past the decode kernel's layout
  int* scratch = tb.misc + 4;   // 32 ints of reduction scratch

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // full: the weight producer's arrival (with its bytes) + 32 token-loader lanes
    for (int i = 0; i < kDecStages; ++i) { mbar_init(&full[i], 33); mbar_init(&empty[i], 16); }
    for (int i = 0; i < kDecUnitRing; ++i) { mbar_init(&ufull[i], 1); mbar_init(&uempty[i], 18); }
    for (int i = 0; i < 2; ++i) { mbar_init(&hpub[i], 512); hcount[i] = 0; }
    *abort_flag = 0;
    tb.misc[kMiscDown] = 0;
    fence_mbarrier_init();
  }
  if (warp == 16 && lane == 0) {
    prefetch_tmap(&tm_c0); prefetch_tmap(&tm_s0); prefetch_tmap(&tm_c1);
    prefetch_tmap(&tm_s1); prefetch_tmap(&tm_c2); prefetch_tmap(&tm_s2);
  }
  if (warp == 17 && lane == 0) prefetch_tmap(&tm_h);
  __syncthreads();
  const Abort ab{abort_flag};

  // the raw slot table, for phase 2a
  for (int e = threadIdx.x; e < p.E; e += blockDim.x) tb.slot[e] = __ldg(p.d.g[0].slot_table + e);

  // ------------------------------------------------------------ phase 1 ---
  // 2T items claimed from a counter: items t < T route token t, items T + t
  // convert row t.  The CTAs that are resident take them all whatever order
  // the grid is scheduled in, so no wait below depends on a CTA that has not
  // started; routing and conversion run on different CTAs at the same time.
  for (;;) {
    if (threadIdx.x == 0) tb.misc[kMiscClaim] = atomicAdd(p.ctrl + 3, 1);
    __syncthreads();
    const int item = tb.misc[kMiscClaim];
    __syncthreads();
    if (item >= 2 * p.T) break;
    if (item < p.T) {
      if (warp == 0) layer_route_token(p, item);
    } else {
      layer_convert_row(p, item - p.T, reinterpret_cast<float*>(scratch));
    }
    // the barrier orders every thread's writes before thread 0's release
    // (cumulative at GPU scope), which publishes them with the count
    __syncthreads();
    if (threadIdx.x == 0) red_release_gpu_add(p.ctrl + (item < p.T ? 0 : 4), 1);
  }
  // ----------------------------------------------------------- phase 2a ---
  const bool counted = layer_counts(p, tb, scratch);
  const int n1 = counted ? tb.misc[0] : 0;
  const int ntot = counted ? tb.misc[1] : 0;
  const int E = p.E;
  // ----------------------------------------------------------- phase 2b ---
  // every warp but the weight producer, which starts streaming meanwhile
  bool sorted = counted;
  if (counted && warp != 16) {
    sorted = layer_scatter(p, tb, kDecThreads - 32, threadIdx.x < 512 ? threadIdx.x : threadIdx.x - 32);
    if (!sorted && threadIdx.x == 0) *abort_flag = 1;
  }

  // ------------------------------------------------------------ phase 3 ---
  if (!counted || (!sorted && warp != 16)) {
    // nothing to do (the status is recorded; the weight producer sees the abort flag)
  } else if (warp == 16) {
    // ------------------------------------------- queue + weight TMA ---
    if (lane == 0) {
      uint32_t si = 0;
      bool ok = true;
      int next_q = atomicAdd(p.ctrl + 1, 1);
      int4 next_raw = next_q < ntot ? layer_unit_desc(p, tb, next_q, n1, E) : make_int4(0, 0, 0, 0);
      for (int j = 0; ok; ++j) {
        const int us = j % kDecUnitRing;
        if (!(ok = ab.wait(&uempty[us], ((j / kDecUnitRing) & 1) ^ 1, kTagUnit, j, -3))) break;
        const int q = next_q < ntot ? next_q : -1;
        const int4 raw = next_raw;
        if (q >= 0) next_q = atomicAdd(p.ctrl + 1, 1);
        udesc[us] = raw;
        uent[us].x = q;
        mbar_arrive(&ufull[us]);
        if (q < 0) break;
        const DecUnit d = decode_unit(p.d, q, n1, raw);
        const DecConsts c = dec_consts(p.d, d);
        const CUtensorMap* c0 = d.gemm ? &tm_c2 : &tm_c0;
        const CUtensorMap* c1 = d.gemm ? &tm_c2 : &tm_c1;
        const CUtensorMap* s0 = d.gemm ? &tm_s2 : &tm_s0;
        const CUtensorMap* s1 = d.gemm ? &tm_s2 : &tm_s1;
        const int y0 = d.gemm ? d.mt * kDecRows : d.mt * kDecFeat1;
        const int y1 = d.gemm ? y0 + 128 : y0;
        for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
          const int s = si % kDecStages;
          if (!(ok = ab.wait(&empty[s], ((si / kDecStages) & 1) ^ 1, kTagWEmpty, si, q))) break;
          if (ws == d.ws1 - 1) uent[us] = make_int4(q, __float_as_int(c.g0), __float_as_int(c.g1), 0);
          mbar_arrive_expect_tx(&full[s], kDecWStageBytes);
          uint8_t* st = smem + s * kDecStageBytes;
          const int tl = p.d.g[0].tiled;
          tma_load_weights(st, c0, &full[s], tl, 128, ws, y0, d.slot);
          tma_load_weights(st + 128 * 128, c1, &full[s], tl, 128, ws, y1, d.slot);
          tma_load_weights(st + kDecCodes, s0, &full[s], tl, 16, ws, y0, d.slot);
          tma_load_weights(st + kDecCodes + 128 * 16, s1, &full[s], tl, 16, ws, y1, d.slot);
        }
        next_raw = next_q < ntot ? layer_unit_desc(p, tb, next_q, n1, E) : make_int4(0, 0, 0, 0);
      }
      dec_drain(full, si);
    }
  } else if (warp == 17) {
    // -------------------------------------- token rows (all 32 lanes) ---
    uint32_t si = 0;
    bool ok = true;
    for (int j = 0; ok; ++j) {
      const int us = j % kDecUnitRing;
      if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -1)))) break;
      const int q = uent[us].x;
      __syncwarp();
      if (q < 0) { if (lane == 0) mbar_arrive(&uempty[us]); break; }
      const DecUnit d = decode_unit(p.d, q, n1, udesc[us]);
      GatherRows gr;
      if (d.gemm == 0) gr = layer_gather_rows(p, tb, d.rb, d.nr, lane);
      if (d.gemm == 1) {
        int okw = 1;
        if (lane == 0) {
          okw = dec_wait_h(p.d, d, ab, q);
          if (okw) fence_proxy_async_global();   // the h rows were written by generic stores
        }
        if (!(ok = __shfl_sync(0xFFFFFFFFu, okw, 0) != 0)) break;
      }
      for (int ws = d.ws0; ws < d.ws1; ++ws, ++si) {
        const int s = si % kDecStages;
        if (!(ok = __all_sync(0xFFFFFFFFu, ab.wait(&empty[s], ((si / kDecStages) & 1) ^ 1, kTagBEmpty, si, q))))
          break;
        uint8_t* bst = smem + s * kDecStageBytes + kDecWStageBytes;
        if (d.gemm == 0) {
          layer_gather_stage(p, gr, bst, &full[s], ws, lane);
        } else {
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[s], kDecBStageBytes);
#pragma unroll
            for (int bx = 0; bx < 4; ++bx)
              tma_load_2d(bst + bx * kDecBBoxBytes, &tm_h, &full[s], ws * kDecStageK + bx * 64, d.rb);
          } else {
            mbar_arrive(&full[s]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[us]);
    }
    cp_async_wait<0>();
    __syncwarp();
    if (lane == 0) dec_drain(full, si);
  } else if (warp == 18) {
    // --------------------------------------------------- publisher ---
    if (lane == 0) {
      int ngu = 0;
      for (int j = 0;; ++j) {
        const int us = j % kDecUnitRing;
        if (!ab.wait(&ufull[us], (j / kDecUnitRing) & 1, kTagUnit, j, -4)) break;
        const int q = uent[us].x;
        if (q < 0) { mbar_arrive(&uempty[us]); break; }
        const DecUnit d = decode_unit(p.d, q, n1, udesc[us]);
        if (d.gemm == 0) {
          const int hb = ngu & 1;
          if (!ab.wait(&hpub[hb], (ngu >> 1) & 1, kTagUnit, ngu, q)) break;
          const int cnt = hcount[hb];
          hcount[hb] = 0;
          if (cnt) {
            fence_proxy_async_global();
            red_release_gpu_add(p.d.tile_done + d.tile, cnt);
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
      const DecUnit d = decode_unit(p.d, q, n1, udesc[us]);
      const int gu = d.gemm == 0 ? ngu++ : -1;
      if (d.gemm == 1 && warp == 0 && lane == 0) ++tb.misc[kMiscDown];
      const bool ok =
          d.nr > 8 ? layer_unit<2, FMT>(p, tb, d, smem, full, empty, ab, &uempty[us], &uent[us], hpub, hcount, gu, si, q, warp, lane)
                   : layer_unit<1, FMT>(p, tb, d, smem, full, empty, ab, &uempty[us], &uent[us], hpub, hcount, gu, si, q, warp, lane);
      if (!ok) break;
    }
  }
  __syncthreads();

  // ------------------------------------------------------------ phase 4 ---
  // The combine, once every down unit of the layer is done: this CTA's down
  // units are published with one release (the barrier above orders all its
  // threads' expert-output stores before it), then every CTA waits until the
  // count reaches the number of down units and sums a strided share of the
  // T x H/4 output vectors -- the combine kernel's arithmetic (fmaf in the
  // order j = 0 .. k-1, each batch's rows and weights requested first), so y
  // is the same bits.  Units are counted, not CTAs, so the wait never depends
  // on a CTA that has not started.
  if (counted && sorted) {
    if (threadIdx.x == 0) {
      red_release_gpu_add(p.ctrl + 5, tb.misc[kMiscDown]);
      tb.misc[kMiscConv] = layer_wait_count(p.ctrl + 5, ntot - n1, kTagCombine) ? 0 : 1;
    }
    __syncthreads();
    if (!tb.misc[kMiscConv]) {
      const int k = p.k, vpr = p.H / 4, P = p.T * k;
      const float4* op = static_cast<const float4*>(p.d.g[1].out);
      float4* y = reinterpret_cast<float4*>(p.y);
      const long long nvec = (long long)p.T * vpr;
      for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < nvec;
           i += (long long)gridDim.x * blockDim.x) {
        const int t = int(i / vpr), c = int(i % vpr);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j0 = 0; j0 < k; j0 += 4) {
          int row[4];
          float wj[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            row[q] = j0 + q < k ? tb.p2r[t * k + j0 + q] : -1;
            wj[q] = j0 + q < k ? tb.w[t * k + j0 + q] : 0.0f;
          }
          float4 o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const bool ok = row[q] >= 0 && row[q] < P;
            if (j0 + q < k && !ok) set_device_status(FT_DEV_BAD_INDEX);
            o[q] = ok ? __ldcg(op + size_t(row[q]) * vpr + c) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (row[q] < 0 || row[q] >= P) continue;
            acc.x = fmaf(wj[q], o[q].x, acc.x);
            acc.y = fmaf(wj[q], o[q].y, acc.y);
            acc.z = fmaf(wj[q], o[q].z, acc.z);
            acc.w = fmaf(wj[q], o[q].w, acc.w);
          }
        }
        y[i] = acc;
      }
    }
  }

  // ------------------------------------------------ end: counter resets ---
  if (threadIdx.x == 0) {
    __threadfence();
    tb.misc[2] = atom_acq_rel_gpu_add(p.ctrl + 2, 1) == int(gridDim.x) - 1;
  }
  __syncthreads();
  if (tb.misc[2]) {   // the last CTA: every other CTA has finished
    const bool dirty = *reinterpret_cast<volatile int*>(&g_device_status) != 0 || !counted;
    const int ntiles = dirty ? p.n_done : tb.misc[3];
    for (int i = threadIdx.x; i < ntiles; i += blockDim.x) p.d.tile_done[i] = 0;
    if (dirty) {
      for (int i = threadIdx.x; i < p.n_cnt1; i += blockDim.x) p.cnt1[i] = 0;
      for (int i = threadIdx.x; i < p.n_cnt2; i += blockDim.x) p.cnt2[i] = 0;
    }
    if (threadIdx.x == 0)
      for (int i = 0; i < kLayerCtrl; ++i) p.ctrl[i] = 0;
  }
}

// ---------------------------------------------------------------- host ---

// The whole-layer call: one launch of layer_decode_kernel when the batch is
// decode-sized (the FFN plan picks the decode variant, T <= 128, T*k <= 1024,
// E <= 512), else the four calls of the separate path on parts of the
// workspace.
struct LayerPlan {
  bool fused;
  FfnPlan ffn;
  // fused: workspace layout (byte offsets)
  size_t off_x16, off_rs, off_h, off_ctrl, off_done, off_cnt1, off_cnt2, off_part1, off_part2;
  int n_done, n_cnt1, n_cnt2;
  // separate calls: permute workspace, then the FFN workspace
  size_t off_perm_ws, off_ffn_ws;
  size_t total;
};

static bool layer_fits(int T, int k, int E, const FfnPlan& f) {
  return f.decode && T >= 1 && T <= kLayerMaxT && T * k <= kLayerMaxP && E <= kLayerMaxE;
}

static LayerPlan plan_layer(int T, int H, int I, int E, int k, int num_sms) {
  LayerPlan L{};
  L.ffn = plan_ffn(T, H, I, E, k, num_sms);
  L.fused = layer_fits(T, k, E, L.ffn);
  const FfnPlan& f = L.ffn;
  const size_t P = size_t(T) * k;
  size_t o = 0;
  if (L.fused) {
    L.off_x16 = o;   o = align256(o + size_t(T) * H * 2);
    L.off_rs = o;    o = align256(o + size_t(T) * 4);
    L.off_h = o;     o = align256(o + P * I * 2);
    L.off_ctrl = o;  o = align256(o + kLayerCtrl * 4);
    L.n_done = int(f.max_tiles1);
    L.off_done = o;  o = align256(o + size_t(L.n_done) * 4);
    L.n_cnt1 = int(f.max_tiles1 * f.mt1 * 16);
    L.off_cnt1 = o;  o = align256(o + size_t(L.n_cnt1) * 4);
    L.n_cnt2 = int(f.max_tiles2 * f.mt2 * 16);
    L.off_cnt2 = o;  o = align256(o + size_t(L.n_cnt2) * 4);
    L.off_part1 = o;
    if (f.g1.splits > 1) o = align256(o + size_t(f.max_units1) * kDecPartialBytes);
    L.off_part2 = o;
    if (f.g2.splits > 1) o = align256(o + size_t(f.max_units2) * kDecPartialBytes);
  } else {
    L.off_perm_ws = o; o = align256(o + permute_ws_bytes(T, k, E));
    L.off_ffn_ws = o;  o = align256(o + f.total);
  }
  L.total = o;
  return L;
}

template <int FMT>
static cudaError_t launch_layer_kernel(const LayerParams& p, int grid, const CUtensorMap (&tmc)[3],
                                       const CUtensorMap (&tms)[3], const CUtensorMap& tm_h, cudaStream_t s) {
  ProfileScope prof(FT_KERNEL_LAYER_DECODE, s);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(layer_decode_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kLayerSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return launch_pdl(layer_decode_kernel<FMT>, dim3(grid), dim3(kDecThreads), kLayerSmemBytes, s, p, tmc[0], tms[0],
                    tmc[1], tms[1], tmc[2], tms[2], tm_h);
}

static cudaError_t launch_layer(const void* x, const float* logits, int T, int H, int I, int E, int k, int mode,
                                const int32_t* slot_table, const void* pool_v, const ft_nvfp4_slot_layout& Ly,
                                int32_t* ids, float* wts, int32_t* offsets, int32_t* perm_src, int32_t* pair_to_row,
                                void* out_perm, void* y, void* ws, cudaStream_t s, const char** why) {
  const int num_sms = device_sm_count();
  const LayerPlan L = plan_layer(T, H, I, E, k, num_sms);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (!L.fused) {
    cudaError_t e = launch_route(logits, T, E, k, mode, ids, wts, s);
    if (e == cudaSuccess) e = launch_permute(ids, T, k, E, offsets, perm_src, pair_to_row, w + L.off_perm_ws, s);
    if (e == cudaSuccess)
      e = launch_ffn(x, T, H, I, E, k, perm_src, offsets, slot_table, pool_v, Ly, out_perm, w + L.off_ffn_ws, s, why);
    if (e == cudaSuccess) e = launch_combine(out_perm, pair_to_row, wts, T, k, H, y, s);
    return e;
  }
  const FfnPlan& pl = L.ffn;
  const uint8_t* pool = static_cast<const uint8_t*>(pool_v);
  CUtensorMap tmc[3], tms[3], tm_h;
  const int rows[3] = {I, I, H}, Ks[3] = {H, H, I};
  for (int m = 0; m < 3; ++m)
    if (!make_weight_maps(pool, Ly, m, rows[m], Ks[m], 128, &tmc[m], &tms[m])) {
      *why = "cuTensorMapEncodeTiled failed for the slot pool";
      return cudaErrorInvalidValue;
    }
  __half* h = reinterpret_cast<__half*>(w + L.off_h);
  if (!make_act_map(h, T * k, I, kDecBN, &tm_h)) {
    *why = "cuTensorMapEncodeTiled failed for h";
    return cudaErrorInvalidValue;
  }
  LayerParams p{};
  FfnParams& p1 = p.d.g[0];
  p1.rowscale = nullptr;   // row factors come from the kernel's own tables
  p1.perm_src = nullptr;
  p1.k_top = k;
  p1.K = H;
  p1.M = I;
  p1.nkw = pl.nkw1;
  p1.nkc = pl.nkc1;
  p1.splits = pl.g1.splits;
  p1.stages_per_split = pl.g1.sps;
  p1.units = nullptr;
  p1.num_units = nullptr;
  p1.slot_table = slot_table;
  p1.pool = pool;
  p1.slot_bytes = Ly.slot_bytes;
  p1.global_off[0] = Ly.global_off[FT_GATE];
  p1.global_off[1] = Ly.global_off[FT_UP];
  p1.out = h;
  p1.partials = reinterpret_cast<float*>(w + L.off_part1);
  p1.counters = reinterpret_cast<int*>(w + L.off_cnt1);
  p1.tiled = Ly.tiled;
  FfnParams& p2 = p.d.g[1];
  p2 = p1;
  p2.K = I;
  p2.M = H;
  p2.nkw = pl.nkw2;
  p2.nkc = pl.nkc2;
  p2.splits = pl.g2.splits;
  p2.stages_per_split = pl.g2.sps;
  p2.global_off[0] = Ly.global_off[FT_DOWN];
  p2.global_off[1] = Ly.global_off[FT_DOWN];
  p2.out = out_perm;
  p2.partials = reinterpret_cast<float*>(w + L.off_part2);
  p2.counters = reinterpret_cast<int*>(w + L.off_cnt2);
  p.d.queue = nullptr;   // the kernel's queue is ctrl[1]
  p.d.tile_done = reinterpret_cast<int*>(w + L.off_done);
  p.d.mt1 = pl.mt1;
  p.d.mt2 = pl.mt2;
  p.logits = logits;
  p.x = static_cast<const uint4*>(x);
  p.T = T; p.E = E; p.k = k; p.H = H; p.mode = mode;
  const int npl = (E + 31) / 32;
  p.npl = npl <= 1 ? 1 : npl <= 2 ? 2 : npl <= 4 ? 4 : npl <= 8 ? 8 : 16;
  p.num_slots = Ly.num_slots;
  p.ids = ids; p.wts = wts; p.offsets = offsets; p.perm_src = perm_src; p.pair_to_row = pair_to_row;
  p.y = static_cast<float*>(y);
  p.x16 = reinterpret_cast<uint4*>(w + L.off_x16);
  p.rowscale = reinterpret_cast<float*>(w + L.off_rs);
  p.ctrl = reinterpret_cast<int*>(w + L.off_ctrl);
  p.tile_done = p.d.tile_done;
  p.cnt1 = p1.counters;
  p.cnt2 = p2.counters;
  p.n_cnt1 = L.n_cnt1; p.n_cnt2 = L.n_cnt2; p.n_done = L.n_done;
  return Ly.scale_format == FT_SCALE_MXFP4 ? launch_layer_kernel<FT_SCALE_MXFP4>(p, num_sms, tmc, tms, tm_h, s)
                                           : launch_layer_kernel<FT_SCALE_NVFP4>(p, num_sms, tmc, tms, tm_h, s);
}

}  // namespace ftmoe
