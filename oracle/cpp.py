"""ctypes front end of the C++ oracle (oracle/moe_oracle.cpp).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Same steps and the same
readings of the pages as the numpy oracle (oracle/moe_layer.py), written
independently; the tests pin both to the hand-worked fixtures and to each
other.
"""
from __future__ import annotations

import ctypes
from ctypes import POINTER, c_double, c_float, c_int, c_int32, c_int64, c_uint8, c_uint16
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_L = None


def lib() -> ctypes.CDLL:
    global _L
    if _L is None:
        L = ctypes.CDLL(_build.build())
        L.orc_e2m1_value.restype = c_double
        L.orc_e2m1_value.argtypes = [c_int]
        L.orc_e4m3_value.restype = c_double
        L.orc_e4m3_value.argtypes = [c_int]
        L.orc_pack.restype = c_int
        L.orc_pack.argtypes = [POINTER(c_float), c_int, c_int, POINTER(c_uint8), POINTER(c_uint8), c_int,
                               POINTER(c_float)]
        L.orc_e8m0_value.restype = c_double
        L.orc_e8m0_value.argtypes = [c_int]
        L.orc_pack_mxfp4.restype = c_int
        L.orc_pack_mxfp4.argtypes = [POINTER(c_float), c_int, c_int, POINTER(c_uint8), POINTER(c_uint8), c_int]
        L.orc_decode_mxfp4.restype = c_int
        L.orc_decode_mxfp4.argtypes = [POINTER(c_uint8), POINTER(c_uint8), c_int, c_int, c_int, POINTER(c_double)]
        L.orc_route.restype = c_int
        L.orc_route.argtypes = [POINTER(c_float), c_int, c_int, c_int, POINTER(c_int32), POINTER(c_double)]
        L.orc_permute.restype = c_int
        L.orc_permute.argtypes = [POINTER(c_int32), c_int, c_int, c_int, POINTER(c_int32), POINTER(c_int32),
                                  POINTER(c_int32)]
        L.orc_moe_layer.restype = c_int
        L.orc_moe_layer.argtypes = [POINTER(c_uint16), POINTER(c_float), c_int, c_int, c_int, c_int, c_int,
                                    POINTER(c_int32), POINTER(c_uint8), c_int64, POINTER(c_int64),
                                    POINTER(c_int64), POINTER(c_int64), POINTER(c_int32), POINTER(c_int32), c_int,
                                    c_int, POINTER(c_double)]
        _L = L
    return _L


def _p(a: np.ndarray, ct):
    return a.ctypes.data_as(POINTER(ct))


def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(code))


def e4m3_value(byte: int) -> float:
    return float(lib().orc_e4m3_value(byte))


def pack(w: np.ndarray, ld_scale: Optional[int] = None):
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    ld = K // 16 if ld_scale is None else ld_scale
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, ld), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    if lib().orc_pack(_p(w, c_float), N, K, _p(codes, c_uint8), _p(scales, c_uint8), ld, _p(g, c_float)) != 0:
        raise ValueError("orc_pack: K must be a multiple of 16 and ld_scale >= K/16")
    return codes, scales, np.float32(g[0])


def e8m0_value(byte: int) -> float:
    return float(lib().orc_e8m0_value(byte))


def pack_mxfp4(w: np.ndarray, ld_scale: Optional[int] = None):
    """fp32 [N, K] -> (codes uint8 [N, K/2], E8M0 scales uint8 [N, ld])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    N, K = w.shape
    ld = K // 32 if ld_scale is None else ld_scale
    codes = np.zeros((N, K // 2), dtype=np.uint8)
    scales = np.zeros((N, ld), dtype=np.uint8)
    rc = lib().orc_pack_mxfp4(_p(w, c_float), N, K, _p(codes, c_uint8), _p(scales, c_uint8), ld)
    if rc != 0:
        raise ValueError({-1: "K must be a multiple of 32 and ld_scale >= K/32",
                          -2: "non-finite input"}.get(rc, str(rc)))
    return codes, scales


def decode_mxfp4(codes: np.ndarray, scales: np.ndarray, K: int) -> np.ndarray:
    """MXFP4 [N, K] -> fp64 values."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N, ld = scales.shape
    out = np.zeros((N, K), dtype=np.float64)
    if lib().orc_decode_mxfp4(_p(codes, c_uint8), _p(scales, c_uint8), N, K, ld, _p(out, c_double)) != 0:
        raise ValueError("orc_decode_mxfp4: bad sizes or a NaN scale byte")
    return out


def route(logits: np.ndarray, k: int):
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), dtype=np.int32)
    w = np.zeros((T, k), dtype=np.float64)
    if lib().orc_route(_p(lg, c_float), T, E, k, _p(ids, c_int32), _p(w, c_double)) != 0:
        raise ValueError("orc_route: need 1 <= k <= E")
    return ids, w


def permute(ids: np.ndarray, E: int):
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T, k = ids.shape
    off = np.zeros(E + 1, dtype=np.int32)
    ps = np.zeros(T * k, dtype=np.int32)
    p2r = np.zeros(T * k, dtype=np.int32)
    if lib().orc_permute(_p(ids, c_int32), T, k, E, _p(off, c_int32), _p(ps, c_int32), _p(p2r, c_int32)) != 0:
        raise ValueError("orc_permute: expert id out of range")
    return off, ps, p2r


def moe_layer(x_bits: np.ndarray, logits: np.ndarray, k: int, slot_table: np.ndarray, pool: np.ndarray,
              slot_bytes: int, codes_off: Sequence[int], scales_off: Sequence[int], global_off: Sequence[int],
              ld_scale: Sequence[int], H: int, I: int, tokens: Optional[Sequence[int]] = None,
              fmt: int = 0) -> np.ndarray:
    """y fp64 [len(tokens), H] (all tokens by default) from a host copy of the slot pool;
    fmt 0: NVFP4 experts, 1: MXFP4 experts."""
    xb = np.ascontiguousarray(x_bits, dtype=np.uint16)
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    tok = np.arange(T, dtype=np.int32) if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    st = np.ascontiguousarray(slot_table, dtype=np.int32)
    pl = np.ascontiguousarray(pool, dtype=np.uint8)
    co = np.asarray(codes_off, dtype=np.int64)
    so = np.asarray(scales_off, dtype=np.int64)
    go = np.asarray(global_off, dtype=np.int64)
    ld = np.asarray(ld_scale, dtype=np.int32)
    y = np.zeros((len(tok), H), dtype=np.float64)
    rc = lib().orc_moe_layer(_p(xb, c_uint16), _p(lg, c_float), T, E, k, H, I, _p(st, c_int32), _p(pl, c_uint8),
                             slot_bytes, _p(co, c_int64), _p(so, c_int64), _p(go, c_int64), _p(ld, c_int32),
                             _p(tok, c_int32), len(tok), int(fmt), _p(y, c_double))
    if rc != 0:
        raise ValueError({-1: "bad argument", -2: "NaN scale byte", -3: "expert not resident"}.get(rc, str(rc)))
    return y
