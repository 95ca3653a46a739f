// The extern "C" boundary of libftmoe.so (declared in include/ftmoe.h):
// argument checks, error reporting and kernel launches.
#include <cstdio>
#include <cstring>
#include <string>

#include "ftmoe.h"

namespace ftmoe {

static thread_local std::string g_last_error;

void set_last_error(const char* msg) { g_last_error = msg ? msg : ""; }

static int fail(int code, const char* what) {
  set_last_error(what);
  return code;
}

static int cuda_fail(cudaError_t e, const char* where) {
  char buf[256];
  std::snprintf(buf, sizeof buf, "%s: %s", where, cudaGetErrorString(e));
  set_last_error(buf);
  return FT_ERR_CUDA;
}

static inline cudaStream_t S(ft_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

}  // namespace ftmoe

using namespace ftmoe;

extern "C" const char* ft_last_error(void) { return g_last_error.c_str(); }

extern "C" const char* ft_version(void) { return "ftmoe 0.1 (sm_100a)"; }

extern "C" int ft_nvfp4_slot_layout_init(int H, int I, int num_slots, ft_nvfp4_slot_layout* out) {
  if (!out || H <= 0 || I <= 0 || H % 64 || I % 64 || num_slots <= 0)
    return fail(FT_ERR_INVALID_ARG, "ft_nvfp4_slot_layout_init: need H, I multiples of 64 and num_slots > 0");
  ft_nvfp4_slot_layout L{};
  L.H = H;
  L.I = I;
  L.num_slots = num_slots;
  const int rows[3] = {I, I, H}, Ks[3] = {H, H, I};
  auto a256 = [](long long v) { return (v + 255) & ~255LL; };
  long long off = 0;
  for (int m = 0; m < 3; ++m) {
    L.ld_scale[m] = ((Ks[m] / 16) + 15) / 16 * 16;
    L.codes_off[m] = off;
    off = a256(off + (long long)rows[m] * (Ks[m] / 2));
    L.scales_off[m] = off;
    off = a256(off + (long long)rows[m] * L.ld_scale[m]);
  }
  for (int m = 0; m < 3; ++m) {
    L.global_off[m] = off + 4 * m;
  }
  off = a256(off + 12);
  L.slot_bytes = off;
  L.scale_format = FT_SCALE_NVFP4;
  *out = L;
  return FT_OK;
}

extern "C" int ft_mxfp4_slot_layout_init(int H, int I, int num_slots, ft_nvfp4_slot_layout* out) {
  const int rc = ft_nvfp4_slot_layout_init(H, I, num_slots, out);
  if (rc == FT_OK) out->scale_format = FT_SCALE_MXFP4;
  return rc;
}

extern "C" int ft_tiled_slot_layout_init(int H, int I, int num_slots, int scale_format, ft_nvfp4_slot_layout* out) {
  if (!out || H <= 0 || I <= 0 || H % 64 || I % 64 || num_slots <= 0 ||
      (scale_format != FT_SCALE_NVFP4 && scale_format != FT_SCALE_MXFP4))
    return fail(FT_ERR_INVALID_ARG, "ft_tiled_slot_layout_init: need H, I multiples of 64, num_slots > 0, a format");
  ft_nvfp4_slot_layout L{};
  L.H = H;
  L.I = I;
  L.num_slots = num_slots;
  const int rows[3] = {I, I, H}, Ks[3] = {H, H, I};
  auto a256 = [](long long v) { return (v + 255) & ~255LL; };
  long long off = 0;
  for (int m = 0; m < 3; ++m) {
    const long long stages = (Ks[m] + 255) / 256;
    L.ld_scale[m] = int(16 * stages);
    L.codes_off[m] = off;
    off = a256(off + stages * rows[m] * 128);
    L.scales_off[m] = off;
    off = a256(off + stages * rows[m] * 16);
  }
  for (int m = 0; m < 3; ++m) L.global_off[m] = off + 4 * m;
  off = a256(off + 12);
  L.slot_bytes = off;
  L.scale_format = scale_format;
  L.tiled = 1;
  *out = L;
  return FT_OK;
}

static bool layout_ok(const ft_nvfp4_slot_layout* L) {
  return L && L->H > 0 && L->I > 0 && L->H % 64 == 0 && L->I % 64 == 0 && L->num_slots >= 1 &&
         L->slot_bytes % 256 == 0 && (L->tiled == 0 || L->tiled == 1) &&
         (L->scale_format == FT_SCALE_NVFP4 || L->scale_format == FT_SCALE_MXFP4);
}

extern "C" int ft_moe_route(const float* logits, int T, int E, int k, int mode, int32_t* ids, float* w,
                            ft_stream_t stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 || (mode != 0 && mode != 1))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_route: need 1 <= k <= min(E, 32), E <= 1024, mode 0 or 1");
  if (T == 0) return FT_OK;
  if (!logits || !ids || !w) return fail(FT_ERR_INVALID_ARG, "ft_moe_route: null pointer");
  const cudaError_t e = launch_route(logits, T, E, k, mode, ids, w, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_route");
}

extern "C" size_t ft_moe_permute_workspace_size(int T, int k, int E) {
  if (T <= 0 || k <= 0 || E <= 0) return 0;
  return permute_ws_bytes(T, k, E);
}

extern "C" int ft_moe_permute(const int32_t* ids, int T, int k, int E, int32_t* offsets, int32_t* perm_src,
                              int32_t* pair_to_row, void* ws, size_t ws_bytes, ft_stream_t stream) {
  if (T < 0 || E < 1 || E > kMaxExperts || k < 1 || k > E || (long long)T * k > (1LL << 30))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_permute: need 1 <= k <= E <= 1024");
  if (!offsets) return fail(FT_ERR_INVALID_ARG, "ft_moe_permute: null pointer");
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(offsets, 0, size_t(E + 1) * sizeof(int32_t), S(stream));
    return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_permute");
  }
  if (!ids || !perm_src || !pair_to_row) return fail(FT_ERR_INVALID_ARG, "ft_moe_permute: null pointer");
  const size_t need = permute_ws_bytes(T, k, E);
  if (need > 0 && (!ws || ws_bytes < need))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_permute: workspace too small");
  const cudaError_t e = launch_permute(ids, T, k, E, offsets, perm_src, pair_to_row, ws, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_permute");
}

extern "C" int ft_moe_route_permute(const float* logits, int T, int E, int k, int mode, int32_t* ids, float* w,
                                    int32_t* offsets, int32_t* perm_src, int32_t* pair_to_row, void* ws,
                                    size_t ws_bytes, ft_stream_t stream) {
  if (T < 0 || E < 1 || E > 1024 || k < 1 || k > E || k > 32 || (mode != 0 && mode != 1) ||
      (long long)T * k > (1LL << 30))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_route_permute: need 1 <= k <= min(E, 32), E <= 1024, mode 0 or 1");
  if (!offsets) return fail(FT_ERR_INVALID_ARG, "ft_moe_route_permute: null pointer");
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(offsets, 0, size_t(E + 1) * sizeof(int32_t), S(stream));
    return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_route_permute");
  }
  if (!logits || !ids || !w || !perm_src || !pair_to_row)
    return fail(FT_ERR_INVALID_ARG, "ft_moe_route_permute: null pointer");
  if (!route_permute_fused_fits(T, k, E)) {
    const int r = ft_moe_route(logits, T, E, k, mode, ids, w, stream);
    return r != FT_OK ? r : ft_moe_permute(ids, T, k, E, offsets, perm_src, pair_to_row, ws, ws_bytes, stream);
  }
  const cudaError_t e =
      launch_route_permute_small(logits, T, E, k, mode, ids, w, offsets, perm_src, pair_to_row, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_route_permute");
}

static bool ffn_shape_ok(int H, int I, int E, int k) {
  return H >= 256 && I >= 256 && H % 64 == 0 && I % 64 == 0 && E >= 1 && E <= 1024 && k >= 1 && k <= E &&
         H <= 65536 && I <= 65536;
}

extern "C" size_t ft_moe_ffn_workspace_size(int T, int H, int I, int E, int k) {
  if (T <= 0 || !ffn_shape_ok(H, I, E, k)) return 0;
  return plan_ffn(T, H, I, E, k, device_sm_count()).total;
}

extern "C" int ft_moe_ffn_nvfp4(const void* x, int T, int H, int I, int E, int k, const int32_t* perm_src,
                                const int32_t* expert_offsets, const int32_t* slot_table, const void* slot_pool,
                                const ft_nvfp4_slot_layout* layout, void* out_perm, void* ws, size_t ws_bytes,
                                ft_stream_t stream) {
  if (T < 0 || !ffn_shape_ok(H, I, E, k))
    return fail(FT_ERR_UNSUPPORTED, "ft_moe_ffn_nvfp4: need H, I >= 256 and multiples of 64, 1 <= k <= E <= 1024");
  if (T == 0) return FT_OK;
  if (!x || !perm_src || !expert_offsets || !slot_table || !slot_pool || !layout || !out_perm || !ws)
    return fail(FT_ERR_INVALID_ARG, "ft_moe_ffn_nvfp4: null pointer");
  if (layout->H != H || layout->I != I || layout->num_slots < 1 || layout->num_slots > (1 << 21) ||
      (layout->tiled != 0 && layout->tiled != 1) ||
      layout->slot_bytes % 256 ||
      (layout->scale_format != FT_SCALE_NVFP4 && layout->scale_format != FT_SCALE_MXFP4))
    return fail(FT_ERR_INVALID_ARG,
                "ft_moe_ffn_nvfp4: layout does not match H, I (or has more than 2^21 slots, or an unknown format)");
  if ((reinterpret_cast<uintptr_t>(slot_pool) & 255) || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(out_perm) & 15))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_ffn_nvfp4: misaligned pointer");
  const FfnPlan pl = plan_ffn(T, H, I, E, k, device_sm_count());
  if (ws_bytes < pl.total) return fail(FT_ERR_INVALID_ARG, "ft_moe_ffn_nvfp4: workspace too small");
  const char* why = "ft_moe_ffn_nvfp4";
  const cudaError_t e = launch_ffn(x, T, H, I, E, k, perm_src, expert_offsets, slot_table, slot_pool, *layout,
                                   out_perm, ws, S(stream), &why);
  return e == cudaSuccess ? FT_OK : cuda_fail(e, why);
}

extern "C" int ft_moe_combine(const void* out_perm, const int32_t* pair_to_row, const float* w, int T, int k,
                              int H, void* y, ft_stream_t stream) {
  if (T < 0 || k < 1 || k > 1024 || H < 4 || H % 4)
    return fail(FT_ERR_INVALID_ARG, "ft_moe_combine: need k >= 1 and H a positive multiple of 4");
  if (T == 0) return FT_OK;
  if (!out_perm || !pair_to_row || !w || !y) return fail(FT_ERR_INVALID_ARG, "ft_moe_combine: null pointer");
  if ((reinterpret_cast<uintptr_t>(out_perm) & 15) || (reinterpret_cast<uintptr_t>(y) & 15))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_combine: out_perm and y must be 16-byte aligned");
  const cudaError_t e = launch_combine(out_perm, pair_to_row, w, T, k, H, y, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_combine");
}

extern "C" size_t ft_moe_layer_workspace_size(int T, int H, int I, int E, int k) {
  if (T <= 0 || !ffn_shape_ok(H, I, E, k)) return 0;
  return plan_layer(T, H, I, E, k, device_sm_count()).total;
}

extern "C" int ft_moe_layer_nvfp4(const void* x, const float* logits, int T, int H, int I, int E, int k, int mode,
                                  const int32_t* slot_table, const void* slot_pool,
                                  const ft_nvfp4_slot_layout* layout, int32_t* ids, float* w, int32_t* offsets,
                                  int32_t* perm_src, int32_t* pair_to_row, void* out_perm, void* y, void* ws,
                                  size_t ws_bytes, ft_stream_t stream) {
  if (T < 0 || !ffn_shape_ok(H, I, E, k) || k > 32 || (mode != FT_ROUTE_SOFTMAX_RENORM && mode != FT_ROUTE_TOPK_SOFTMAX))
    return fail(FT_ERR_UNSUPPORTED,
                "ft_moe_layer_nvfp4: need H, I >= 256 and multiples of 64, 1 <= k <= min(E, 32), E <= 1024, a mode");
  if (!offsets) return fail(FT_ERR_INVALID_ARG, "ft_moe_layer_nvfp4: null pointer");
  const cudaStream_t s = S(stream);
  if (T == 0) {
    const cudaError_t e = cudaMemsetAsync(offsets, 0, size_t(E + 1) * sizeof(int32_t), s);
    return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_moe_layer_nvfp4");
  }
  if (!x || !logits || !slot_table || !slot_pool || !layout || !ids || !w || !perm_src || !pair_to_row ||
      !out_perm || !y || !ws)
    return fail(FT_ERR_INVALID_ARG, "ft_moe_layer_nvfp4: null pointer");
  if (layout->H != H || layout->I != I || layout->num_slots < 1 || layout->num_slots > (1 << 21) ||
      (layout->tiled != 0 && layout->tiled != 1) || layout->slot_bytes % 256 ||
      (layout->scale_format != FT_SCALE_NVFP4 && layout->scale_format != FT_SCALE_MXFP4))
    return fail(FT_ERR_INVALID_ARG,
                "ft_moe_layer_nvfp4: layout does not match H, I (or has more than 2^21 slots, or an unknown format)");
  if ((reinterpret_cast<uintptr_t>(slot_pool) & 255) || (reinterpret_cast<uintptr_t>(ws) & 255) ||
      (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(out_perm) & 15) ||
      (reinterpret_cast<uintptr_t>(y) & 15))
    return fail(FT_ERR_INVALID_ARG, "ft_moe_layer_nvfp4: misaligned pointer");
  if (ws_bytes < plan_layer(T, H, I, E, k, device_sm_count()).total)
    return fail(FT_ERR_INVALID_ARG, "ft_moe_layer_nvfp4: workspace too small");
  const char* why = "ft_moe_layer_nvfp4";
  const cudaError_t e = launch_layer(x, logits, T, H, I, E, k, mode, slot_table, slot_pool, *layout, ids, w, offsets,
                                     perm_src, pair_to_row, out_perm, y, ws, s, &why);
  return e == cudaSuccess ? FT_OK : cuda_fail(e, why);
}

extern "C" int ft_gather_rows(const void* src, int n_src, int row_bytes, const int32_t* idx, int div, int n,
                              void* dst, ft_stream_t stream) {
  if (n < 0 || n_src < 0 || row_bytes < 16 || row_bytes % 16 || div < 1)
    return fail(FT_ERR_INVALID_ARG, "ft_gather_rows: need n, n_src >= 0, row_bytes a positive multiple of 16, div >= 1");
  if (n == 0) return FT_OK;
  if (!src || !idx || !dst) return fail(FT_ERR_INVALID_ARG, "ft_gather_rows: null pointer");
  if ((reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
    return fail(FT_ERR_INVALID_ARG, "ft_gather_rows: src and dst must be 16-byte aligned");
  const cudaError_t e = launch_gather_rows(src, n_src, row_bytes, idx, div, n, dst, device_sm_count(), S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_gather_rows");
}

extern "C" int ft_nvfp4_pack(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld_scale,
                             float* global_scale, void* ws, ft_stream_t stream) {
  if (N < 1 || K < 16 || K % 16 || ld_scale < K / 16)
    return fail(FT_ERR_INVALID_ARG, "ft_nvfp4_pack: need N >= 1, K a multiple of 16, ld_scale >= K/16");
  if (!w || !codes || !scales || !global_scale || !ws) return fail(FT_ERR_INVALID_ARG, "ft_nvfp4_pack: null pointer");
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(codes) & 7) || ((K / 2) % 8))
    return fail(FT_ERR_INVALID_ARG, "ft_nvfp4_pack: w must be 16-byte and codes 8-byte aligned");
  const cudaError_t e =
      launch_pack(w, N, K, row_major_place(codes, scales, K, ld_scale), ld_scale, global_scale, ws, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_nvfp4_pack");
}

extern "C" int ft_pack_slot(const float* w, int mat, const ft_nvfp4_slot_layout* L, void* slot, void* ws,
                            ft_stream_t stream) {
  if (!layout_ok(L) || mat < 0 || mat > 2)
    return fail(FT_ERR_INVALID_ARG, "ft_pack_slot: bad layout or tensor index");
  if (!w || !slot || !ws) return fail(FT_ERR_INVALID_ARG, "ft_pack_slot: null pointer");
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(slot) & 255))
    return fail(FT_ERR_INVALID_ARG, "ft_pack_slot: w must be 16-byte and the slot 256-byte aligned");
  const int N = mat == FT_DOWN ? L->H : L->I, K = mat == FT_DOWN ? L->I : L->H;
  uint8_t* base = static_cast<uint8_t*>(slot);
  PackPlace pl;
  pl.codes = base + L->codes_off[mat];
  pl.scales = base + L->scales_off[mat];
  pl.tiled = L->tiled;
  pl.c_row = L->tiled ? 128 : K / 2;
  pl.c_stage = L->tiled ? 128LL * N : 128;
  pl.s_row = L->tiled ? 16 : L->ld_scale[mat];
  pl.s_stage = L->tiled ? 16LL * N : 16;
  float* g = reinterpret_cast<float*>(base + L->global_off[mat]);
  const cudaError_t e = L->scale_format == FT_SCALE_MXFP4
                            ? launch_pack_mxfp4(w, N, K, pl, L->ld_scale[mat], g, ws, S(stream))
                            : launch_pack(w, N, K, pl, L->ld_scale[mat], g, ws, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_pack_slot");
}

extern "C" int ft_mxfp4_pack(const float* w, int N, int K, uint8_t* codes, uint8_t* scales, int ld_scale,
                             float* global_scale, void* ws, ft_stream_t stream) {
  if (N < 1 || K < 16 || K % 32 || ld_scale < K / 16)
    return fail(FT_ERR_INVALID_ARG, "ft_mxfp4_pack: need N >= 1, K a multiple of 32, ld_scale >= K/16");
  if (!w || !codes || !scales || !global_scale || !ws) return fail(FT_ERR_INVALID_ARG, "ft_mxfp4_pack: null pointer");
  if ((reinterpret_cast<uintptr_t>(w) & 15) || (reinterpret_cast<uintptr_t>(codes) & 7) || ((K / 2) % 8))
    return fail(FT_ERR_INVALID_ARG, "ft_mxfp4_pack: w must be 16-byte and codes 8-byte aligned");
  const cudaError_t e = launch_pack_mxfp4(w, N, K, row_major_place(codes, scales, K, ld_scale), ld_scale,
                                          global_scale, ws, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_mxfp4_pack");
}

extern "C" int ft_device_status(int* status, int clear) {
  if (!status) return fail(FT_ERR_INVALID_ARG, "ft_device_status: null pointer");
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "ft_device_status");
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "ft_device_status");
  if (clear) {
    const int zero = 0;
    const long long zeros[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    e = cudaMemcpyToSymbol(g_device_status_detail, zeros, sizeof(zeros));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "ft_device_status");
  }
  *status = v;
  return FT_OK;
}

extern "C" int ft_selftest_wait_timeout(int32_t* out, ft_stream_t stream) {
  if (!out) return fail(FT_ERR_INVALID_ARG, "ft_selftest_wait_timeout: null pointer");
  const cudaError_t e = launch_wait_selftest(out, S(stream));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_selftest_wait_timeout");
}

extern "C" int ft_device_status_detail(int64_t* detail) {
  if (!detail) return fail(FT_ERR_INVALID_ARG, "ft_device_status_detail: null pointer");
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(detail, g_device_status_detail, 8 * sizeof(long long));
  return e == cudaSuccess ? FT_OK : cuda_fail(e, "ft_device_status_detail");
}

extern "C" int ft_profile_enable(int on) {
  profiler().enabled.store(on ? 1 : 0);
  return FT_OK;
}

extern "C" int ft_profile_read(ft_profile_t* out, int reset) {
  if (!out) return fail(FT_ERR_INVALID_ARG, "ft_profile_read: null pointer");
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  std::memset(out, 0, sizeof(*out));
  for (int k = 0; k < FT_KERNEL_KINDS; ++k) out->launches[k] = P.launches[k].load();
  for (auto& r : P.pending) {
    float ms = 0.0f;
    if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) {
      out->timed[r.kind] += 1;
      out->total_ms[r.kind] += ms;
    }
  }
  if (reset) {
    for (auto& r : P.pending) { P.spare.push_back(r.a); P.spare.push_back(r.b); }
    P.pending.clear();
    for (auto& l : P.launches) l = 0;
  }
  return FT_OK;
}
