/*
 * ftmoe.h -- C ABI of libftmoe.so: one Mixture-of-Experts FFN layer over
 * NVFP4-quantised experts, for NVIDIA B200 (sm_100a).
 *
 * The layer is the hot path of the MoE serving engine described on the
 * FreeToken pages ("FlashML-org / FreeToken" About page, "Fast Edge-Native
 * Runtime": MoE serving with a global LRU expert cache and graph-compatible
 * execution; "FreeToken model guide", MoE expert scheduling strategies and
 * --quant-backend moe.nvfp4; "sm89-moe-offload" fork README, "Production
 * configuration" with --moe-cache-size and the wide-load NVFP4 prefill MoE
 * kernel).  The pages name the pieces but never write the layer down; the
 * operations below are the plainest reading of a top-k MoE FFN layer:
 *
 *   route    -> ft_moe_route      top-k over fp32 router logits, renormalised weights
 *   permute  -> ft_moe_permute    pairs grouped per expert, expert offsets
 *   experts  -> ft_moe_ffn_nvfp4  h = silu(Wg x) * (Wu x), o = Wd h, per group
 *   combine  -> ft_moe_combine    y[t] = sum_j w[t,j] * o[row(t,j)]
 *   format   -> ft_nvfp4_pack     fp32 weights -> NVFP4 (E2M1 + E4M3/16 + fp32)
 *   cache    -> ft_slot_*         host LRU of expert slots in a device pool
 *   EP       -> ft_ep_plan, ft_gather_rows   experts split over ranks; the rows
 *                                 of each rank's experts exchanged all-to-all
 *
 * Conventions (all functions):
 *   - Return an int status (FT_OK or a negative FT_ERR_*).  On FT_ERR_CUDA the
 *     message of the failing runtime call is in ft_last_error() (per thread).
 *   - Device pointers are plain device addresses; the caller owns every
 *     buffer (device memory, pinned host memory, workspaces).  No function
 *     allocates device memory on the hot path.
 *   - Device work is enqueued on the caller's stream and returns without
 *     synchronising, except ft_slot_acquire (host LRU bookkeeping) and
 *     ft_device_status (reads a device word).  Enqueued work never reads the
 *     host and never synchronises, so a sequence of calls can be captured in
 *     a CUDA graph.
 *   - T = 0 is a valid no-op.
 *   - Kernels never trap: a bad index or an over-long internal wait records
 *     a code in a per-device status word (FT_DEV_*) and the kernel returns;
 *     read and clear it with ft_device_status.
 */
#ifndef FTMOE_H_
#define FTMOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FT_API __attribute__((visibility("default")))
#else
#define FT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ft_stream_t; /* a cudaStream_t; NULL = legacy default stream */

enum {
  FT_OK = 0,
  FT_ERR_INVALID_ARG = -1,  /* null pointer, k > E, k > 32, E > 1024, bad size or leading dim */
  FT_ERR_UNSUPPORTED = -2,  /* a shape outside what the kernels support */
  FT_ERR_CUDA = -3,         /* a CUDA runtime error; see ft_last_error() */
  FT_ERR_CAPACITY = -4,     /* the slot pool cannot hold the experts one call needs */
  FT_ERR_NOT_RESIDENT = -5, /* an expert has no host bank registered */
  FT_ERR_DEVICE = -6,       /* the device status word was set by a kernel */
};

/* Device status codes recorded by kernels (read with ft_device_status). */
enum {
  FT_DEV_OK = 0,
  FT_DEV_WAIT_TIMEOUT = 1,  /* an internal pipeline wait exceeded ~1 s */
  FT_DEV_NOT_RESIDENT = 2,  /* a non-empty expert group had slot -1 */
  FT_DEV_BAD_INDEX = 3,     /* an expert id or slot outside its range */
  FT_DEV_F16_RANGE = 4,     /* an intermediate exceeded the f16 range (saturated) */
};

enum {
  FT_ROUTE_SOFTMAX_RENORM = 0, /* softmax over all E logits, keep top-k, renormalise */
  FT_ROUTE_TOPK_SOFTMAX = 1,   /* keep top-k logits, softmax over those k */
};

enum { FT_GATE = 0, FT_UP = 1, FT_DOWN = 2 };

/*
 * Where one expert's three NVFP4 tensors live inside a slot of the device
 * pool (pool + slot * slot_bytes + offset).  Gate and up are [I, H], down is
 * [H, I] (row = output feature, K contiguous).  For a tensor [N, K]:
 *   codes   uint8 [N, K/2]       two E2M1 codes per byte, even k in the low nibble
 *   scales  uint8 [N, ld_scale]  one E4M3 (FN) byte per 16 consecutive k
 *   global  fp32                 per-tensor scale
 * value(n,k) = e2m1(code) * e4m3(scale[n][k/16]) * global.
 * ld_scale is K/16 rounded up to a multiple of 16; all offsets and
 * slot_bytes are multiples of 256.
 */
typedef struct {
  int32_t H, I;
  int32_t ld_scale[3];    /* bytes per scale row of gate, up, down */
  int64_t codes_off[3];
  int64_t scales_off[3];
  int64_t global_off[3];
  int64_t slot_bytes;
  int32_t num_slots;      /* slots in the pool the layout describes */
  int32_t scale_format;   /* FT_SCALE_NVFP4 or FT_SCALE_MXFP4 */
  int32_t tiled;          /* 0: codes [N, K/2] and scales [N, ld_scale] row-major;
                             1: stage-tiled (see ft_tiled_slot_layout_init) */
} ft_nvfp4_slot_layout;

/* How a slot's scale bytes and global scales read.
 *   FT_SCALE_NVFP4: one E4M3 scale per 16 K of a row; the tensor's fp32
 *                   global scale multiplies every value.
 *   FT_SCALE_MXFP4: one E8M0 scale 2^(s - 127) per 32 K of a row (OCP MX),
 *                   stored twice (as if per 16 K) so that both formats share
 *                   every offset and stride; the global holds a power of two
 *                   2^t chosen at pack time, which the kernels divide out of
 *                   the dequantised values and multiply back in fp32 (the
 *                   values are e2m1 * 2^(s - 127), the global only keeps the
 *                   f16 dequantisation exact). */
enum { FT_SCALE_NVFP4 = 0, FT_SCALE_MXFP4 = 1 };

/* Fill *out with the canonical layout for hidden size H, intermediate I and
 * num_slots slots.  H and I must be multiples of 64.  Returns FT_OK or
 * FT_ERR_INVALID_ARG. */
FT_API int ft_nvfp4_slot_layout_init(int H, int I, int num_slots, ft_nvfp4_slot_layout* out);
/* The same layout with scale_format = FT_SCALE_MXFP4 (identical offsets). */
FT_API int ft_mxfp4_slot_layout_init(int H, int I, int num_slots, ft_nvfp4_slot_layout* out);
/*
 * A stage-tiled slot layout (tiled = 1) in either scale format.  The same
 * bytes are arranged so that what the expert GEMMs load together is
 * contiguous: for a tensor [N, K] with S = ceil(K / 256) stages of 256 K,
 *   codes   uint8 [S][N][128]  byte (s, n, j) holds k = 256 s + 2 j, 2 j + 1
 *   scales  uint8 [S][N][16]   byte (s, n, j) is the scale of k / 16 = 16 s + j
 * so one stage of 128 rows is one 16 KB block of codes and one 2 KB block of
 * scales.  Bytes past K/2 in the last stage hold zero codes.  ld_scale
 * (= 16 S) and the global offsets keep their meaning.
 */
FT_API int ft_tiled_slot_layout_init(int H, int I, int num_slots, int scale_format,
                                     ft_nvfp4_slot_layout* out);

/*
 * Pack fp32 weights w [N, K] (device; N, K the shape of tensor `mat` of the
 * layout) into the tensor's place in one slot (slot: device address of the
 * slot's first byte), in the layout's scale format and arrangement: the
 * arithmetic of ft_nvfp4_pack or ft_mxfp4_pack, the bytes placed as the
 * layout says.  ws as for those calls.
 */
FT_API int ft_pack_slot(const float* w, int mat, const ft_nvfp4_slot_layout* layout, void* slot, void* ws,
                        ft_stream_t stream);

/*
 * Router: per token t, the k experts with the largest logits (descending;
 * equal logits -> lower expert id first) and their renormalised weights
 *   w_j = exp(l_j - m) / sum_{i in S} exp(l_i - m),  m = max over S.
 * mode selects how the fp32 arithmetic is ordered (FT_ROUTE_*); the selected
 * ids never depend on it.
 *   logits    device fp32 [T, E] row-major
 *   topk_ids  device int32 [T, k]  (out)
 *   topk_w    device fp32  [T, k]  (out)
 * Requires 1 <= k <= min(E, 32), E <= 1024.
 * Pages: the routers of the MoE families in "FreeToken model guide" (its
 * model table: Qwen3.6-35B-A3B, gpt-oss, Gemma-4 A4B and the like) and the
 * "MoE serving" of the About page's "Fast Edge-Native Runtime" select k
 * experts per token; no page writes the router down, so the two weightings
 * (softmax over all experts then renormalised over the k, or softmax over
 * the k) are this library's reading of a top-k router.
 */
FT_API int ft_moe_route(const float* logits, int T, int E, int k, int mode,
                 int32_t* topk_ids, float* topk_w, ft_stream_t stream);

/*
 * Permute: pair p = t*k + j (routed to expert topk_ids[p]) is given row
 * r = expert_offsets[e] + (rank of p among the pairs of e, ascending p).
 *   expert_offsets  device int32 [E+1]  exclusive prefix sum of group sizes (out)
 *   perm_src        device int32 [T*k]  row -> pair (out)
 *   pair_to_row     device int32 [T*k]  pair -> row (out)
 *   ws              device workspace of ft_moe_permute_workspace_size bytes
 * Deterministic (no atomics decide any order).  Ids outside [0, E) set
 * FT_DEV_BAD_INDEX.
 * Pages: the grouping of tokens per expert that a grouped expert GEMM needs
 * (the "sm89-moe-offload" fork README, "Key customizations": the NVFP4
 * prefill MoE kernel for M >= 2048 rows) is not described on any page; a
 * stable counting sort by expert is the plainest reading.  Determinism
 * follows the About page's "graph-compatible execution" ("Fast Edge-Native
 * Runtime"): the same inputs replay to the same bytes.
 */
FT_API int ft_moe_permute(const int32_t* topk_ids, int T, int k, int E,
                   int32_t* expert_offsets, int32_t* perm_src, int32_t* pair_to_row,
                   void* ws, size_t ws_bytes, ft_stream_t stream);
FT_API size_t ft_moe_permute_workspace_size(int T, int k, int E);

/*
 * ft_moe_route followed by ft_moe_permute, as one call: the outputs of both,
 * bit for bit.  Small batches (T <= 128, T*k <= 1024, E <= 512: the decode
 * sizes) run both steps in one kernel launch that keeps the selected ids in
 * shared memory; other sizes launch the two calls' kernels.  Arguments are
 * those of the two calls; ws and ws_bytes as for ft_moe_permute (no
 * workspace is needed when T*k <= 1024).
 */
FT_API int ft_moe_route_permute(const float* logits, int T, int E, int k, int mode,
                                int32_t* topk_ids, float* topk_w, int32_t* expert_offsets,
                                int32_t* perm_src, int32_t* pair_to_row, void* ws, size_t ws_bytes,
                                ft_stream_t stream);

/*
 * ft_moe_permute without a workspace argument and without allocating.  The
 * pages have no counterpart of this call: it is an interface convenience.
 * Output is identical, bit for bit, to ft_moe_permute's.
 *
 * It is meant for callers that cannot draw device memory when they call:
 * a host program with no device allocator, or a runtime whose device memory
 * is all partitioned at start-up.  The per-chunk counts go to a fixed
 * 256 KiB array inside this library, which limits inputs to
 * ceil(T*k / 1024) * E <= 65536 (always met when T*k <= 1024); larger inputs
 * return FT_ERR_INVALID_ARG and launch nothing.  The array needs no zeroing.
 *
 * Every call looks up the current device's copy of the array (a host-side
 * query, valid across devices and after a device reset); the first call on
 * a device may load the library's device code there, so make it before any
 * stream capture.  Calls on one device share the array: two calls that can
 * overlap in time (different streams, or different host threads) race and
 * give wrong rows, so order them.
 * Arguments are those of ft_moe_permute minus ws and ws_bytes.
 */
FT_API int ft_moe_permute_noalloc(const int32_t* topk_ids, int T, int k, int E,
                   int32_t* expert_offsets, int32_t* perm_src, int32_t* pair_to_row,
                   ft_stream_t stream);

/*
 * Expert FFN over the permuted rows.  For row r of group e (token
 * t = perm_src[r] / k), with the expert's tensors at
 * slot_pool + slot_table[e] * layout->slot_bytes:
 *   h[r]        = silu(gG * (Qg x_t)) * (gU * (Qu x_t))        (I values)
 *   out_perm[r] = gD * (Qd h[r])                                (H values, fp32)
 * where Q* are the E2M1*E4M3 dequantised weights, g* the fp32 global scales,
 * and products accumulate in fp32 on the tensor cores.  The MMA operands are
 * f16:
 *   - every E2M1*E4M3 product is exact in f16;
 *   - each token row x_t is converted once, times the power of two 2^(12-e)
 *     that puts its largest magnitude in [2^13, 2^15) (e = 0 when max|x_t| is
 *     in [2, 8), else max|x_t| * 2^-e is in [4, 8); any finite bf16 row has
 *     one).  Elements within a factor 2^30 of the row's largest magnitude
 *     convert exactly; smaller ones round with an absolute error of at most
 *     2^-38 max|x_t|;
 *   - h is rounded to f16 after dividing it by 2^(2e), the square of its
 *     row's factor (undone exactly, in fp32, on the down projection's
 *     output), so its range does not depend on the row's magnitude, only
 *     on the weights and the row's shape.  A normalised h beyond +-65504
 *     saturates and sets FT_DEV_F16_RANGE.
 * The expert outputs stay fp32 so that the layer output meets
 * |y - y_exact| <= 1e-2 rms(y) + 1e-3: a bf16 rounding of them (or of y) alone
 * would already reach that bound at the tails of the output distribution.
 *   x              device bf16 [T, H]
 *   perm_src       device int32 [T*k]     from ft_moe_permute
 *   expert_offsets device int32 [E+1]     from ft_moe_permute
 *   slot_table     device int32 [E]       expert -> slot; -1 = not resident
 *   slot_pool      device, layout->num_slots * layout->slot_bytes bytes, 256-B aligned
 *   out_perm       device fp32 [T*k, H]   (out)
 *   ws             device workspace of ft_moe_ffn_workspace_size bytes, 256-B aligned
 * A non-empty group whose slot is -1 sets FT_DEV_NOT_RESIDENT and its rows are
 * left unwritten.  H and I must be multiples of 64 and match the layout.
 * Pages: NVFP4 expert weights and their MoE kernels ("FreeToken model
 * guide", the NVFP4 releases of each family and --quant-backend
 * moe.nvfp4=marlin|b12x|triton; the "sm89-moe-offload" fork README,
 * "Production configuration" and "Key customizations": the wide-load NVFP4
 * prefill MoE kernel, prior art for sm_89); experts addressed through the
 * expert cache (About page, "Fast Edge-Native Runtime": global LRU expert
 * caching).  The SwiGLU expert (silu(gate) * up, then down) is the expert
 * of the MoE families the model guide lists; no page writes it down.
 */
FT_API int ft_moe_ffn_nvfp4(const void* x, int T, int H, int I, int E, int k,
                     const int32_t* perm_src, const int32_t* expert_offsets,
                     const int32_t* slot_table, const void* slot_pool,
                     const ft_nvfp4_slot_layout* layout,
                     void* out_perm, void* ws, size_t ws_bytes, ft_stream_t stream);
FT_API size_t ft_moe_ffn_workspace_size(int T, int H, int I, int E, int k);

/*
 * Combine: y[t, :] = sum_{j<k} topk_w[t,j] * out_perm[pair_to_row[t*k+j], :],
 * summed in fp32 in the order j = 0..k-1.
 *   out_perm device fp32 [T*k, H], pair_to_row device int32 [T*k],
 *   topk_w device fp32 [T, k], y device fp32 [T, H] (out).  H % 4 == 0;
 *   out_perm and y 16-byte aligned.
 * Pages: the weighted return of each token's k expert outputs is the last
 * step of the "MoE serving" of the About page ("Fast Edge-Native Runtime");
 * no page writes it down, and the fixed summation order is this library's
 * reading of its "graph-compatible execution" (replays give the same bytes).
 */
FT_API int ft_moe_combine(const void* out_perm, const int32_t* pair_to_row, const float* topk_w,
                   int T, int k, int H, void* y, ft_stream_t stream);

/*
 * The whole layer -- route, permute, experts, combine -- as one call, with
 * the outputs of the four calls above, bit for bit:
 *   ft_moe_route(logits, T, E, k, mode, topk_ids, topk_w)
 *   ft_moe_permute(topk_ids, T, k, E, expert_offsets, perm_src, pair_to_row)
 *   ft_moe_ffn_nvfp4(x, T, H, I, E, k, perm_src, expert_offsets, slot_table, slot_pool, layout, out_perm)
 *   ft_moe_combine(out_perm, pair_to_row, topk_w, T, k, H, y)
 * (the steps of the layer as the pages' serving engine runs it: top-k router,
 * grouping of the tokens per expert, NVFP4 expert FFNs, weighted sum;
 * "FlashML-org / FreeToken" About page, "Fast Edge-Native Runtime", and the
 * FreeToken model guide's MoE expert scheduling section).
 *
 * Decode-sized batches (few token rows per expert, T <= 128, T*k <= 1024,
 * E <= 512) run all of it in ONE persistent kernel launch: the grid routes
 * the tokens, every CTA sorts the pairs in its own shared memory, the expert
 * GEMMs stream the weights as ft_moe_ffn_nvfp4 does, and the combine runs
 * inside the down GEMM's epilogue.  Other sizes make the four calls.
 *
 * Arguments are those of the four calls (same layouts, same alignment
 * rules); x bf16 [T, H], logits fp32 [T, E], y fp32 [T, H].
 *   ws   device workspace of ft_moe_layer_workspace_size bytes, 256-B aligned.
 *        It must be zero-filled once before its first use (cudaMemset); each
 *        call leaves it ready for the next, including a call that recorded a
 *        device status.  One workspace serves one call at a time.
 * A token whose experts include a non-resident one (slot -1) gets no y row
 * (FT_DEV_NOT_RESIDENT is recorded).
 */
FT_API int ft_moe_layer_nvfp4(const void* x, const float* logits, int T, int H, int I, int E, int k, int mode,
                              const int32_t* slot_table, const void* slot_pool,
                              const ft_nvfp4_slot_layout* layout, int32_t* topk_ids, float* topk_w,
                              int32_t* expert_offsets, int32_t* perm_src, int32_t* pair_to_row, void* out_perm,
                              void* y, void* ws, size_t ws_bytes, ft_stream_t stream);
FT_API size_t ft_moe_layer_workspace_size(int T, int H, int I, int E, int k);

/*
 * NVFP4 pack of one fp32 tensor [N, K] (K % 16 == 0), every step an IEEE fp32
 * operation rounded to nearest:
 *   g   = amax / 2688 (1 if amax = 0)                  -> *global_scale
 *   s_b = E4M3_rne_sat(amax_b / (6 g))                  per 16-block of a row
 *   q   = E2M1_rne_sat(w / (e4m3(s_b) * g))             0 where e4m3(s_b) = 0
 * Ties go to the even code; the code's sign bit follows the input's sign.
 *   w            device fp32 [N, K]
 *   codes        device uint8 [N, K/2]       (out; row pitch K/2)
 *   scales       device uint8 [N, ld_scale]  (out; padding bytes zeroed)
 *   global_scale device fp32 [1]             (out)
 *   ws           device workspace, >= 4 bytes (holds amax)
 * The destinations may point inside a slot (see ft_nvfp4_slot_layout).
 * Pages: NVFP4 is the expert format of the served checkpoints ("FreeToken
 * model guide", the -NVFP4 releases and --quant-backend moe.nvfp4; the
 * "sm89-moe-offload" fork README, "Production configuration"; About page,
 * "Broad MoE & Ecosystem Support": MXFP4, NVFP4, FP8, BF16).  No page defines
 * the format's bits; the layout above is NVIDIA's published NVFP4 (E2M1
 * values, one E4M3 scale per 16, an fp32 tensor scale), and the choice of g
 * (amax / (6 * 448)) is this library's reading.
 */
FT_API int ft_nvfp4_pack(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld_scale,
                  float* global_scale, void* ws, ft_stream_t stream);

/*
 * MXFP4 pack of one fp32 tensor [N, K] (K % 32 == 0): the OCP Microscaling
 * (MX) conversion, which the pages name as an expert format beside NVFP4
 * ("FlashML-org / FreeToken" About page, "Broad MoE & Ecosystem Support") without
 * defining it.  Per 32-block b of a row:
 *   x_b = floor(log2 amax_b) - 2, clamped to [-127, 127]; -127 if amax_b = 0
 *   scale byte s_b = x_b + 127, written at scales[row][2b] and [2b + 1]
 *   q   = E2M1_rne_sat(w / 2^x_b), sign following w
 * and for the tensor t = max_b x_b - 13 (0 if the tensor is all zero):
 *   *global_scale = 2^t  (so that every e2m1 * 2^(x_b - t) the kernels form
 *                         in f16 stays below 2^16; a block more than 2^36
 *                         below the tensor's largest would lose values to f16
 *                         underflow: the kernel then records FT_DEV_F16_RANGE)
 * Arguments as for ft_nvfp4_pack (ld_scale >= K/16: the scales are stored at
 * the NVFP4 granularity).  Returns FT_OK, FT_ERR_INVALID_ARG or FT_ERR_CUDA.
 */
FT_API int ft_mxfp4_pack(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld_scale,
                  float* global_scale, void* ws, ft_stream_t stream);

/*
 * Read (and optionally clear) the per-device status word of the current
 * device.  Synchronises the device.  *status receives an FT_DEV_* code.
 */
FT_API int ft_device_status(int* status, int clear);

/*
 * Where the first recorded device status came from (synchronises the
 * device): detail[0] code, [1] block, [2] warp, [3] barrier kind (for a wait
 * timeout: 1 weight-stage free, 2 weight-stage full, 3 token-stage free,
 * 4 token-stage full, 5 operand-slot free, 6 operand-slot full,
 * 7 accumulator free, 8 accumulator full), [4] the waiting role's counter,
 * [5] work unit, [6] microseconds waited, [7] reserved.  Cleared together
 * with the status word by ft_device_status(..., clear = 1).
 */
FT_API int ft_device_status_detail(int64_t detail[8]);

/*
 * Test hook for the failure path: launches one CTA of two warps that wait on
 * mbarriers nothing completes, through the bounded wait of the expert
 * GEMMs.  Warp 0's wait gives up after ~1 s and records FT_DEV_WAIT_TIMEOUT
 * (detail: block 0, warp 0, barrier kind 4, counter 7, unit 3) and raises
 * the CTA's abort flag; warp 1, which starts 0.5 s later, sees the flag and
 * leaves before its own limit.  out[w] (device int32 [2]) = 1 when warp w's
 * wait gave up.  The kernel ends normally (no trap, no fault), so the
 * context stays usable.  Takes one to two seconds of device time.
 */
FT_API int ft_selftest_wait_timeout(int32_t* out, ft_stream_t stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism.  The fork's production configuration splits the experts
 * of every MoE layer over two GPUs ("sm89-moe-offload" fork README,
 * "Production configuration": --moe-ep-size 2 beside tensor parallelism);
 * the pages do not say how the rows travel.  The reading used here, for G
 * ranks with E % G == 0:
 *   - rank r owns experts [r*E/G, (r+1)*E/G) (contiguous blocks);
 *   - every rank routes and permutes its own T_r tokens over all E experts,
 *     so the rows it must send to rank d are one contiguous range of its
 *     permuted rows: [offsets_r[d*E/G], offsets_r[(d+1)*E/G]);
 *   - the ranks exchange their expert_offsets (an all-gather of G x (E+1)
 *     int32), then all-to-all the activation rows (ft_gather_rows with
 *     idx = perm_src, div = k lays them out), run ft_moe_ffn_nvfp4 over their
 *     own experts on what arrived, all-to-all the output rows back, and
 *     combine as on one GPU.
 * Rows arrive grouped by source rank; the plan gives the receiver a
 * perm_src that visits them expert by expert, so the FFN reads them in
 * place (x = the received rows, T = n_recv, k = 1, E = E/G), and the inverse
 * map to put the outputs back in arrival order (ft_gather_rows, div = 1).
 * Each rank's out_perm then holds, row for row, what one GPU would compute.
 * ------------------------------------------------------------------------- */

/*
 * The exchange plan of `rank`, on the host (no CUDA calls).
 *   all_offsets     host int32 [G][E+1]: every rank's expert_offsets from
 *                   ft_moe_permute (row s from rank s); each row starts at 0
 *                   and never decreases
 *   send_rows       host int32 [G] (out): rows this rank sends to rank d
 *   recv_rows       host int32 [G] (out): rows it receives from rank s
 *   local_offsets   host int32 [E/G + 1] (out): group offsets of its experts
 *                   over the received rows, expert by expert
 *   perm_src_local  host int32 [cap] (out): row r of that grouping -> index of
 *                   the received row (arrival order: by source rank, then as
 *                   the source's permuted order); within an expert, rows go
 *                   by source rank, then by the source's pair order
 *   ret_idx         host int32 [cap] (out): the inverse of perm_src_local
 *   *n_recv         (out) rows received = local_offsets[E/G]
 * perm_src_local and ret_idx may both be NULL (sizes only).  Returns
 * FT_ERR_INVALID_ARG for G < 1, E % G != 0, rank outside [0, G), malformed
 * offsets, or n_recv > cap (after writing *n_recv and the row counts).
 */
FT_API int ft_ep_plan(const int32_t* all_offsets, int G, int E, int rank, int32_t* send_rows,
                      int32_t* recv_rows, int32_t* local_offsets, int32_t* perm_src_local,
                      int32_t* ret_idx, int cap, int32_t* n_recv);

/*
 * Row gather on the device: dst[i, :] = src[idx[i] / div, :] for i in [0, n).
 *   src        device, n_src rows of row_bytes bytes
 *   idx        device int32 [n]
 *   dst        device, n rows of row_bytes bytes (out)
 * row_bytes must be a positive multiple of 16 and src and dst 16-byte
 * aligned; div >= 1.  An index whose row falls outside [0, n_src) sets
 * FT_DEV_BAD_INDEX and gives a zero row.  n = 0 is a no-op.
 */
FT_API int ft_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx, int div, int n,
                          void* dst, ft_stream_t stream);

/* ---------------------------------------------------------------------------
 * Expert slot manager: a host-side LRU over (layer, expert) keys, mirroring
 * the pages' global LRU expert cache (FreeToken model guide, offload strategy,
 * OffloadMoeCache with per-(layer, expert) recency and a minimum-size guard;
 * sm89-moe-offload README, --moe-cache-size).  Each registered expert has a
 * pinned host copy of its slot image (layout->slot_bytes bytes); the misses of
 * one call are filled on the caller's copy stream, one cudaMemcpyAsync per run
 * of consecutive slots whose host copies are consecutive too (register the
 * banks of a layer in one page-locked block to get long runs), and the
 * compute stream waits on an event recorded after the copies.
 * ------------------------------------------------------------------------- */
typedef struct ft_slot_mgr ft_slot_mgr;

typedef struct {
  int64_t hits, misses, evictions, bytes_h2d;
  int64_t copies;   /* cudaMemcpyAsync calls the fills took (runs of consecutive slots and banks) */
} ft_slot_stats_t;

enum {
  FT_SLOT_DEVICE = 0,    /* normal mode: fills and table uploads on the copy stream */
  FT_SLOT_HOST_ONLY = 1, /* bookkeeping only: no CUDA calls, device_slot_table is host
                            memory; for planning and for testing the policy on a host */
};

/* Manage slots [0, capacity) of device_pool (capacity <= layout->num_slots).
 * device_pool may be NULL with FT_SLOT_HOST_ONLY. */
FT_API int ft_slot_create(ft_slot_mgr** mgr, int capacity, const ft_nvfp4_slot_layout* layout,
                   void* device_pool, int flags);
/* pinned_src: page-locked host memory of slot_bytes bytes, owned by the caller
 * and kept alive while the manager exists. */
FT_API int ft_slot_register_host(ft_slot_mgr* mgr, int layer, int expert, const void* pinned_src);
/*
 * Make the n experts host_expert_ids[0..n) of `layer` resident and write
 * device_slot_table[e] (an int32 [E] device array, E = table_len) for them;
 * other entries are set to -1.  Resident experts of this call are pinned
 * until the next acquire; misses evict the least recently used unpinned
 * slots.  Returns FT_ERR_CAPACITY when more distinct experts are requested
 * than the pool can hold, FT_ERR_NOT_RESIDENT when a miss has no host bank.
 * The bookkeeping is synchronous on the host; the fills and the table upload
 * are enqueued on `copy` and `compute` waits for them.  A fill that reuses a
 * slot first waits (on `copy`) for the compute work that last read that slot:
 * the work enqueued on `compute` before the acquire that followed the one
 * which handed the slot out.  So the fills of the next layer overlap the
 * current layer's kernels.  The host blocks only when the table upload of
 * eight calls earlier is still pending (a ring of page-locked staging
 * buffers).  device_slot_table must not be read by kernels still in flight
 * when it is passed again: use one table per layer in flight.
 */
FT_API int ft_slot_acquire(ft_slot_mgr* mgr, int layer, const int32_t* host_expert_ids, int n,
                    int32_t* device_slot_table, int table_len, ft_stream_t compute, ft_stream_t copy);
FT_API int ft_slot_stats(const ft_slot_mgr* mgr, ft_slot_stats_t* out);
FT_API int ft_slot_destroy(ft_slot_mgr* mgr);
/* Test hook: make the next `count` host->device fills fail (FT_ERR_CUDA). */
FT_API int ft_slot_inject_copy_failures(ft_slot_mgr* mgr, int count);

/* ---------------------------------------------------------------------------
 * Launch accounting and kernel timing.  Every kernel the library launches is
 * counted by kind.  With timing enabled, CUDA events are recorded around each
 * launch on its stream (not while the stream is being captured into a graph).
 * ------------------------------------------------------------------------- */
enum {
  FT_KERNEL_ROUTE = 0,
  FT_KERNEL_PERMUTE = 1,
  FT_KERNEL_SCHEDULE = 2,     /* (work lists; now built inside the FT_KERNEL_PREP launch) */
  FT_KERNEL_GEMM_GATE_UP = 3, /* grouped gate/up GEMM + SwiGLU */
  FT_KERNEL_GEMM_DOWN = 4,    /* grouped down GEMM */
  FT_KERNEL_COMBINE = 5,
  FT_KERNEL_PACK = 6,
  FT_KERNEL_PREP = 7,         /* work lists + activations to f16 (inside ft_moe_ffn_nvfp4) */
  FT_KERNEL_FFN_DECODE = 8,   /* decode variant: gate/up + SwiGLU + down in one launch */
  FT_KERNEL_GATHER = 9,       /* row gather of the expert-parallel exchange */
  FT_KERNEL_ROUTE_PERMUTE = 10, /* route and permute in one launch (small batches) */
  FT_KERNEL_LAYER_DECODE = 11,  /* the whole layer in one launch (ft_moe_layer_nvfp4, small batches) */
  FT_KERNEL_KINDS = 12,
};

typedef struct {
  int64_t launches[FT_KERNEL_KINDS];   /* launches since the last reset */
  int64_t timed[FT_KERNEL_KINDS];      /* launches that were timed */
  double total_ms[FT_KERNEL_KINDS];    /* summed device time of the timed launches */
} ft_profile_t;

/* Turn event timing on (1) or off (0). */
FT_API int ft_profile_enable(int on);
/* Synchronise the recorded events, fill *out, and optionally reset. */
FT_API int ft_profile_read(ft_profile_t* out, int reset);

/* Message of the last FT_ERR_* returned on this thread ("" if none). */
FT_API const char* ft_last_error(void);

/* Library version string. */
FT_API const char* ft_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FTMOE_H_ */
