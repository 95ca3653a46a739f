"""The C-ABI library loads, exports every function include/ftmoe.h declares,
and rejects bad arguments before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from moe_expert_layer_renorm_b200 import _lib
from moe_expert_layer_renorm_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build()
    return _lib.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "ftmoe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*FT_API\s+(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s*(ft_[a-z0-9_]+)\s*\(", src,
                       flags=re.M)
    return sorted(set(names))


def test_header_declares_the_hot_path_calls():
    names = declared_functions()
    for required in ("ft_moe_route", "ft_moe_permute", "ft_moe_ffn_nvfp4", "ft_moe_combine", "ft_nvfp4_pack",
                     "ft_slot_create", "ft_slot_acquire", "ft_slot_destroy", "ft_last_error"):
        assert required in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_ctypes_signatures_cover_the_header():
    assert set(declared_functions()) <= set(_lib._SIGS)


def test_version(L):
    assert "sm_100a" in _lib.version()


def test_slot_layout_rules(L):
    for H, I in ((256, 512), (2048, 768), (2048, 512), (2880, 2880), (320, 448)):
        lay = _lib.slot_layout(H, I, 7)
        rows = (I, I, H)
        ks = (H, H, I)
        ends = []
        for m in range(3):
            assert lay.ld_scale[m] % 16 == 0 and lay.ld_scale[m] >= ks[m] // 16
            assert lay.codes_off[m] % 256 == 0 and lay.scales_off[m] % 256 == 0
            assert lay.codes_off[m] + rows[m] * ks[m] // 2 <= lay.scales_off[m]
            ends.append(lay.scales_off[m] + rows[m] * lay.ld_scale[m])
        assert lay.codes_off[1] >= ends[0] and lay.codes_off[2] >= ends[1]
        assert min(lay.global_off) >= ends[2]
        assert lay.slot_bytes % 256 == 0 and lay.slot_bytes >= max(lay.global_off) + 4
        assert lay.num_slots == 7
    # 2880/16 = 180 scale bytes per row, padded to 192 for 16-byte TMA rows
    assert _lib.slot_layout(2880, 2880, 1).ld_scale[0] == 192


def test_slot_layout_rejects_bad_sizes(L):
    with pytest.raises(_lib.FtError) as ei:
        _lib.slot_layout(100, 512, 1)
    assert ei.value.code == _lib.FT_ERR_INVALID_ARG


def test_argument_checks_need_no_gpu(L):
    # k > E
    assert L.ft_moe_route(None, 4, 8, 9, 0, None, None, None) == _lib.FT_ERR_INVALID_ARG
    assert b"k <=" in L.ft_last_error()
    # E > 1024
    assert L.ft_moe_route(None, 4, 2000, 2, 0, None, None, None) == _lib.FT_ERR_INVALID_ARG
    # T == 0 is a no-op
    assert L.ft_moe_route(None, 0, 8, 2, 0, None, None, None) == _lib.FT_OK
    assert L.ft_moe_combine(None, None, None, 0, 2, 256, None, None) == _lib.FT_OK
    assert L.ft_moe_combine(None, None, None, 4, 2, 250, None, None) == _lib.FT_ERR_INVALID_ARG
    lay = _lib.slot_layout(256, 512, 8)
    # unsupported sizes
    assert L.ft_moe_ffn_nvfp4(None, 4, 192, 512, 8, 2, None, None, None, None, ctypes.byref(lay), None, None, 0,
                              None) == _lib.FT_ERR_UNSUPPORTED
    # null pointers
    assert L.ft_moe_ffn_nvfp4(None, 4, 256, 512, 8, 2, None, None, None, None, ctypes.byref(lay), None, None, 0,
                              None) == _lib.FT_ERR_INVALID_ARG
    assert L.ft_nvfp4_pack(None, 4, 20, None, None, 2, None, None, None) == _lib.FT_ERR_INVALID_ARG


def test_workspace_queries(L):
    assert _lib.permute_workspace_size(16, 2, 8) == 0            # one chunk: no workspace
    assert _lib.permute_workspace_size(8192, 10, 512) == 80 * 512 * 4
    small = _lib.ffn_workspace_size(16, 256, 512, 8, 2)
    big = _lib.ffn_workspace_size(4096, 2048, 768, 128, 8)
    assert small > 16 * 2 * 512 * 2 and big > 4096 * 8 * 768 * 2
    assert _lib.ffn_workspace_size(0, 2048, 768, 128, 8) == 0


@pytest.mark.parametrize("H,I", [(256, 512), (2048, 768), (2880, 2880), (320, 448)])
def test_reference_layout_matches_library(H, I):
    import bench
    ref = bench.reference_layout(H, I)
    L = _lib.slot_layout(H, I, 3)
    assert list(L.ld_scale) == ref["ld_scale"] and list(L.codes_off) == ref["codes_off"]
    assert list(L.scales_off) == ref["scales_off"] and list(L.global_off) == ref["global_off"]
    assert L.slot_bytes == ref["slot_bytes"]


def test_argument_checks_of_the_later_entry_points(L):
    # route + permute in one call: the route rules, and T == 0 needs offsets only
    assert L.ft_moe_route_permute(None, 4, 8, 9, 0, None, None, None, None, None, None, 0, None) \
        == _lib.FT_ERR_INVALID_ARG
    assert L.ft_moe_route_permute(None, 4, 8, 2, 2, None, None, None, None, None, None, 0, None) \
        == _lib.FT_ERR_INVALID_ARG                                       # mode 2
    assert L.ft_moe_route_permute(None, 0, 8, 2, 0, None, None, None, None, None, None, 0, None) \
        == _lib.FT_ERR_INVALID_ARG                                       # no offsets to clear
    assert b"null" in L.ft_last_error()
    # row gather: row length a positive multiple of 16 bytes, div >= 1; n == 0 is a no-op
    assert L.ft_gather_rows(None, 4, 24, None, 1, 4, None, None) == _lib.FT_ERR_INVALID_ARG
    assert L.ft_gather_rows(None, 4, 32, None, 0, 4, None, None) == _lib.FT_ERR_INVALID_ARG
    assert L.ft_gather_rows(None, 4, 32, None, 1, 4, None, None) == _lib.FT_ERR_INVALID_ARG   # null pointers
    assert L.ft_gather_rows(None, 4, 32, None, 1, 0, None, None) == _lib.FT_OK
    assert L.ft_selftest_wait_timeout(None, None) == _lib.FT_ERR_INVALID_ARG
    # MXFP4 pack: K a multiple of 32
    assert L.ft_mxfp4_pack(None, 4, 48, None, None, 16, None, None, None) == _lib.FT_ERR_INVALID_ARG


def test_mxfp4_layout_is_the_nvfp4_layout_with_its_tag(L):
    a, b = _lib.slot_layout(2048, 768, 5), _lib.slot_layout(2048, 768, 5, _lib.FT_SCALE_MXFP4)
    assert (a.scale_format, b.scale_format) == (_lib.FT_SCALE_NVFP4, _lib.FT_SCALE_MXFP4)
    for f in ("ld_scale", "codes_off", "scales_off", "global_off"):
        assert list(getattr(a, f)) == list(getattr(b, f))
    assert a.slot_bytes == b.slot_bytes


@pytest.mark.parametrize("H,I", [(256, 512), (2048, 768), (2880, 2880), (320, 448)])
@pytest.mark.parametrize("fmt", [0, 1])
def test_tiled_layout_rules(L, H, I, fmt):
    lay = _lib.slot_layout(H, I, 3, fmt, tiled=True)
    rows = (I, I, H)
    ks = (H, H, I)
    assert (lay.tiled, lay.scale_format, lay.num_slots) == (1, fmt, 3)
    ends = []
    for m in range(3):
        S = (ks[m] + 255) // 256
        assert lay.ld_scale[m] == 16 * S
        assert lay.codes_off[m] % 256 == 0 and lay.scales_off[m] % 256 == 0
        assert lay.codes_off[m] + S * rows[m] * 128 <= lay.scales_off[m]
        ends.append(lay.scales_off[m] + S * rows[m] * 16)
    assert lay.codes_off[1] >= ends[0] and lay.codes_off[2] >= ends[1]
    assert min(lay.global_off) >= ends[2] and lay.slot_bytes % 256 == 0
    # when every K is a multiple of 256 the tiled slot has the row-major slot's size
    if H % 256 == 0 and I % 256 == 0:
        assert lay.slot_bytes == _lib.slot_layout(H, I, 3, fmt).slot_bytes


def test_pack_slot_argument_checks(L):
    lay = _lib.slot_layout(256, 512, 2, 0, tiled=True)
    assert L.ft_pack_slot(None, 0, ctypes.byref(lay), None, None, None) == _lib.FT_ERR_INVALID_ARG
    assert L.ft_pack_slot(None, 3, ctypes.byref(lay), None, None, None) == _lib.FT_ERR_INVALID_ARG
    bad = _lib.slot_layout(256, 512, 2)
    bad.tiled = 2
    assert L.ft_pack_slot(None, 0, ctypes.byref(bad), None, None, None) == _lib.FT_ERR_INVALID_ARG
    assert L.ft_tiled_slot_layout_init(256, 512, 2, 5, ctypes.byref(bad)) == _lib.FT_ERR_INVALID_ARG


def test_untile_reads_stage_tiled_bytes_back_row_major():
    from moe_expert_layer_renorm_b200.layer import untile
    g = np.random.default_rng(3)
    for N, K in ((5, 2880), (3, 512), (1, 64)):
        S = (K + 255) // 256
        rows = g.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
        tiled = np.zeros((S, N, 128), np.uint8)
        for n in range(N):             # by the definition: byte j of row n goes to stage j // 128, column j % 128
            for j in range(K // 2):
                tiled[j // 128, n, j % 128] = rows[n, j]
        assert np.array_equal(untile(tiled.reshape(-1), N, 128, K // 2), rows)
