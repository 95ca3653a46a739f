"""ctypes binding of libftmoe.so (declared in include/ftmoe.h).

Argument marshalling only: every function forwards plain pointers and sizes
to the C ABI.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint8, c_void_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libftmoe.so")

FT_OK = 0
FT_ERR_INVALID_ARG = -1
FT_ERR_UNSUPPORTED = -2
FT_ERR_CUDA = -3
FT_ERR_CAPACITY = -4
FT_ERR_NOT_RESIDENT = -5
FT_ERR_DEVICE = -6

FT_DEV_OK = 0
FT_DEV_WAIT_TIMEOUT = 1
FT_DEV_NOT_RESIDENT = 2
FT_DEV_BAD_INDEX = 3
FT_DEV_F16_RANGE = 4

FT_ROUTE_SOFTMAX_RENORM = 0
FT_ROUTE_TOPK_SOFTMAX = 1
FT_GATE, FT_UP, FT_DOWN = 0, 1, 2
FT_SLOT_DEVICE = 0
FT_SLOT_HOST_ONLY = 1


class FtError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"ftmoe error {code}: {msg}")
        self.code = code


class SlotLayout(ctypes.Structure):
    _fields_ = [
        ("H", c_int32), ("I", c_int32),
        ("ld_scale", c_int32 * 3),
        ("codes_off", c_int64 * 3),
        ("scales_off", c_int64 * 3),
        ("global_off", c_int64 * 3),
        ("slot_bytes", c_int64),
        ("num_slots", c_int32),
        ("scale_format", c_int32),
        ("tiled", c_int32),
    ]


FT_KERNEL_NAMES = ("route", "permute", "schedule", "gemm_gate_up", "gemm_down", "combine", "pack", "prep_x",
                   "ffn_decode", "gather", "route_permute", "layer_decode")


class Profile(ctypes.Structure):
    _fields_ = [("launches", c_int64 * len(FT_KERNEL_NAMES)), ("timed", c_int64 * len(FT_KERNEL_NAMES)),
                ("total_ms", ctypes.c_double * len(FT_KERNEL_NAMES))]


class SlotStats(ctypes.Structure):
    _fields_ = [("hits", c_int64), ("misses", c_int64), ("evictions", c_int64), ("bytes_h2d", c_int64),
                ("copies", c_int64)]


_SIGS = {
    "ft_nvfp4_slot_layout_init": (c_int, [c_int, c_int, c_int, POINTER(SlotLayout)]),
    "ft_mxfp4_slot_layout_init": (c_int, [c_int, c_int, c_int, POINTER(SlotLayout)]),
    "ft_tiled_slot_layout_init": (c_int, [c_int, c_int, c_int, c_int, POINTER(SlotLayout)]),
    "ft_pack_slot": (c_int, [c_void_p, c_int, POINTER(SlotLayout), c_void_p, c_void_p, c_void_p]),
    "ft_moe_route": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "ft_moe_permute": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                               c_void_p]),
    "ft_moe_permute_workspace_size": (c_size_t, [c_int, c_int, c_int]),
    "ft_moe_route_permute": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                     c_void_p, c_void_p, c_size_t, c_void_p]),
    "ft_moe_permute_noalloc": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "ft_moe_ffn_nvfp4": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                 c_void_p, POINTER(SlotLayout), c_void_p, c_void_p, c_size_t, c_void_p]),
    "ft_moe_ffn_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "ft_moe_combine": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_void_p]),
    "ft_moe_layer_nvfp4": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                   POINTER(SlotLayout), c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                   c_void_p, c_void_p, c_size_t, c_void_p]),
    "ft_moe_layer_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int]),
    "ft_nvfp4_pack": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p]),
    "ft_mxfp4_pack": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p]),
    "ft_device_status": (c_int, [POINTER(c_int), c_int]),
    "ft_device_status_detail": (c_int, [POINTER(c_int64)]),
    "ft_selftest_wait_timeout": (c_int, [c_void_p, c_void_p]),
    "ft_gather_rows": (c_int, [c_void_p, c_int, c_int, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "ft_ep_plan": (c_int, [POINTER(c_int32), c_int, c_int, c_int, POINTER(c_int32), POINTER(c_int32),
                           POINTER(c_int32), POINTER(c_int32), POINTER(c_int32), c_int, POINTER(c_int32)]),
    "ft_slot_create": (c_int, [POINTER(c_void_p), c_int, POINTER(SlotLayout), c_void_p, c_int]),
    "ft_slot_register_host": (c_int, [c_void_p, c_int, c_int, c_void_p]),
    "ft_slot_acquire": (c_int, [c_void_p, c_int, POINTER(c_int32), c_int, c_void_p, c_int, c_void_p, c_void_p]),
    "ft_slot_stats": (c_int, [c_void_p, POINTER(SlotStats)]),
    "ft_slot_destroy": (c_int, [c_void_p]),
    "ft_slot_inject_copy_failures": (c_int, [c_void_p, c_int]),
    "ft_profile_enable": (c_int, [c_int]),
    "ft_profile_read": (c_int, [POINTER(Profile), c_int]),
    "ft_last_error": (c_char_p, []),
    "ft_version": (c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m moe_expert_layer_renorm_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def check(code: int) -> None:
    if code != FT_OK:
        raise FtError(code, lib().ft_last_error().decode())


FT_SCALE_NVFP4, FT_SCALE_MXFP4 = 0, 1


def slot_layout(H: int, I: int, num_slots: int, fmt: int = FT_SCALE_NVFP4, tiled: bool = False) -> SlotLayout:
    L = SlotLayout()
    if tiled:
        check(lib().ft_tiled_slot_layout_init(H, I, num_slots, fmt, ctypes.byref(L)))
        return L
    init = lib().ft_mxfp4_slot_layout_init if fmt == FT_SCALE_MXFP4 else lib().ft_nvfp4_slot_layout_init
    check(init(H, I, num_slots, ctypes.byref(L)))
    return L


def pack_slot(w, mat, layout: SlotLayout, slot, ws, stream) -> None:
    check(lib().ft_pack_slot(w, mat, ctypes.byref(layout), slot, ws, stream))


def route(logits, T, E, k, mode, ids, w, stream) -> None:
    check(lib().ft_moe_route(logits, T, E, k, mode, ids, w, stream))


def permute_workspace_size(T, k, E) -> int:
    return int(lib().ft_moe_permute_workspace_size(T, k, E))


def permute(ids, T, k, E, offsets, perm_src, pair_to_row, ws, ws_bytes, stream) -> None:
    check(lib().ft_moe_permute(ids, T, k, E, offsets, perm_src, pair_to_row, ws, ws_bytes, stream))


def route_permute(logits, T, E, k, mode, ids, w, offsets, perm_src, pair_to_row, ws, ws_bytes, stream) -> None:
    check(lib().ft_moe_route_permute(logits, T, E, k, mode, ids, w, offsets, perm_src, pair_to_row, ws, ws_bytes,
                                     stream))


def permute_noalloc(ids, T, k, E, offsets, perm_src, pair_to_row, stream) -> None:
    """ft_moe_permute without a workspace: for callers that cannot allocate
    device memory at call time (limits and sharing rules in the C header)."""
    check(lib().ft_moe_permute_noalloc(ids, T, k, E, offsets, perm_src, pair_to_row, stream))


def ffn_workspace_size(T, H, I, E, k) -> int:
    return int(lib().ft_moe_ffn_workspace_size(T, H, I, E, k))


def ffn_nvfp4(x, T, H, I, E, k, perm_src, offsets, slot_table, pool, layout, out_perm, ws, ws_bytes,
              stream) -> None:
    check(lib().ft_moe_ffn_nvfp4(x, T, H, I, E, k, perm_src, offsets, slot_table, pool, ctypes.byref(layout),
                                 out_perm, ws, ws_bytes, stream))


def combine(out_perm, pair_to_row, w, T, k, H, y, stream) -> None:
    check(lib().ft_moe_combine(out_perm, pair_to_row, w, T, k, H, y, stream))


def layer_workspace_size(T, H, I, E, k) -> int:
    return int(lib().ft_moe_layer_workspace_size(T, H, I, E, k))


def layer_nvfp4(x, logits, T, H, I, E, k, mode, slot_table, pool, layout, ids, w, offsets, perm_src, pair_to_row,
                out_perm, y, ws, ws_bytes, stream) -> None:
    check(lib().ft_moe_layer_nvfp4(x, logits, T, H, I, E, k, mode, slot_table, pool, ctypes.byref(layout), ids, w,
                                   offsets, perm_src, pair_to_row, out_perm, y, ws, ws_bytes, stream))


def gather_rows(src, n_src, row_bytes, idx, div, n, dst, stream) -> None:
    check(lib().ft_gather_rows(src, n_src, row_bytes, idx, div, n, dst, stream))


def ep_plan(all_offsets, G: int, E: int, rank: int, cap: int, send_rows, recv_rows, local_offsets,
            perm_src_local, ret_idx) -> int:
    """ft_ep_plan on host int32 arrays (numpy or CPU torch, C-contiguous);
    perm_src_local and ret_idx may both be None.  Returns n_recv."""
    def p(a):
        return None if a is None else ctypes.cast(a.ctypes.data if hasattr(a, "ctypes") else a.data_ptr(),
                                                  POINTER(c_int32))
    n = c_int32(0)
    check(lib().ft_ep_plan(p(all_offsets), G, E, rank, p(send_rows), p(recv_rows), p(local_offsets),
                           p(perm_src_local), p(ret_idx), cap, ctypes.byref(n)))
    return int(n.value)


def nvfp4_pack(w, N, K, codes, scales, ld_scale, global_scale, ws, stream) -> None:
    check(lib().ft_nvfp4_pack(w, N, K, codes, scales, ld_scale, global_scale, ws, stream))


def mxfp4_pack(w, N, K, codes, scales, ld_scale, global_scale, ws, stream) -> None:
    check(lib().ft_mxfp4_pack(w, N, K, codes, scales, ld_scale, global_scale, ws, stream))


def device_status(clear: bool = True) -> int:
    v = c_int(0)
    check(lib().ft_device_status(ctypes.byref(v), 1 if clear else 0))
    return v.value


def selftest_wait_timeout(out, stream) -> None:
    """ft_selftest_wait_timeout: a kernel whose bounded waits run out (~1 s)."""
    check(lib().ft_selftest_wait_timeout(out, stream))


def device_status_detail() -> list:
    d = (c_int64 * 8)()
    check(lib().ft_device_status_detail(d))
    return [int(v) for v in d]


def profile_enable(on: bool) -> None:
    check(lib().ft_profile_enable(1 if on else 0))


def profile_read(reset: bool = True) -> dict:
    """{kernel kind: (launches, timed launches, total device ms)}"""
    p = Profile()
    check(lib().ft_profile_read(ctypes.byref(p), 1 if reset else 0))
    return {n: (int(p.launches[i]), int(p.timed[i]), float(p.total_ms[i])) for i, n in enumerate(FT_KERNEL_NAMES)}


def version() -> str:
    return lib().ft_version().decode()
