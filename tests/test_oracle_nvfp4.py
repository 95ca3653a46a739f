"""Pins for the oracle's NVFP4 format code (decode and pack).

Each check compares the oracle with something other than itself: hand-worked
fixtures under tests/golden/, torch's own float8_e4m3fn and bfloat16 casts,
and brute-force nearest-value searches.
"""
import math

import numpy as np
import pytest
import torch

from oracle import nvfp4
from tests.conftest import golden_lines


def test_e2m1_table_matches_hand_worked_fixture():
    rows = golden_lines("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        got = nvfp4.e2m1_value(int(code))
        assert got == float(val)
        assert math.copysign(1.0, got) == math.copysign(1.0, float(val))  # -0 keeps its sign


def test_e4m3_spot_values_hand_worked():
    for byte, val in golden_lines("e4m3_spot.txt"):
        got = nvfp4.e4m3_value(int(byte, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)


def test_e4m3_all_codes_match_torch_float8():
    raw = torch.arange(256, dtype=torch.uint8)
    ref = raw.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nvfp4.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(ours))
    assert np.array_equal(ref[~nan], ours[~nan])
    assert nan.sum() == 2  # 0x7f and 0xff


def test_every_e2m1_e4m3_product_is_exact_in_bf16():
    q = nvfp4.E2M1_TABLE
    s = nvfp4.E4M3_TABLE[~np.isnan(nvfp4.E4M3_TABLE)]
    prod = np.outer(q, s).reshape(-1)
    assert prod.size == 16 * 254
    rt = torch.from_numpy(prod).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(rt, prod)
    nz = np.abs(prod[prod != 0])
    assert nz.min() == 2.0 ** -10 and nz.max() == 2688.0


def test_e2m1_rounding_hand_worked():
    for v, code in golden_lines("e2m1_rounding.txt"):
        assert int(nvfp4.e2m1_rne_sat(np.array([float(v)], np.float32))[0]) == int(code), v


def test_e4m3_rounding_matches_torch_cast():
    g = np.random.default_rng(7)
    v = np.concatenate([
        g.uniform(0, 448, 20000), g.uniform(0, 0.05, 20000), np.exp(g.uniform(-12, 6, 20000)),
        nvfp4.E4M3_TABLE[:127],                                    # exact codes
        (nvfp4.E4M3_TABLE[:126] + nvfp4.E4M3_TABLE[1:127]) / 2,    # exact midpoints
    ]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ours = nvfp4.e4m3_rne_sat(v.astype(np.float64))
    assert np.array_equal(ours, ref)


def test_e4m3_rounding_saturates():
    assert int(nvfp4.e4m3_rne_sat(np.array([448.0]))[0]) == 0x7E
    assert int(nvfp4.e4m3_rne_sat(np.array([1e6]))[0]) == 0x7E


def _brute_nearest(v, grid):
    """Nearest grid index by exhaustive search; ties -> even index."""
    best = None
    for i, gv in enumerate(grid):
        d = abs(v - gv)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    return best[1]


def test_grid_rounding_brute_force():
    g = np.random.default_rng(3)
    grid = nvfp4.E2M1_TABLE[:8]
    for v in np.concatenate([g.uniform(0, 7, 300), (grid[1:] + grid[:-1]) / 2, grid]):
        expect = _brute_nearest(min(v, 6.0), grid)
        assert nvfp4.e2m1_rne_sat(np.array([v], np.float32))[0] == expect


def test_pack_hand_worked_example():
    w = np.zeros((2, 32), np.float32)
    codes = np.zeros((2, 32), np.int64)
    scales = np.zeros((2, 2), np.int64)
    gexp = None
    for row in golden_lines("pack_worked.txt"):
        if row[0] == "w":
            w[int(row[1])] = [float(x) for x in row[2:]]
        elif row[0] == "codes":
            codes[int(row[1])] = [int(x) for x in row[2:]]
        elif row[0] == "scales":
            scales[int(row[1])] = [int(x, 16) for x in row[2:]]
        elif row[0] == "global":
            gexp = float(row[1])
    packed, sc, g = nvfp4.pack(w)
    assert float(g) == gexp
    assert np.array_equal(sc, scales)
    assert np.array_equal(nvfp4.unpack_codes(packed, 2, 32), codes)


def test_pack_all_zero_tensor():
    packed, sc, g = nvfp4.pack(np.zeros((3, 48), np.float32), ld_scale=16)
    assert float(g) == 1.0 and not packed.any() and not sc.any() and sc.shape == (3, 16)


def test_pack_nibble_order_even_k_low():
    w = np.zeros((1, 16), np.float32)
    w[0, 0] = 6.0          # amax -> code 7 at k = 0
    w[0, 1] = -6.0         # code 15 at k = 1
    packed, _, _ = nvfp4.pack(w)
    assert packed[0, 0] == 0xF7


def test_pack_roundtrip_and_error_bound():
    g = np.random.default_rng(11)
    N, K = 64, 256
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[3, 16:32] = 0.0                        # a zero block
    w[5, :16] *= 1e-6                        # a tiny block (scale underflows)
    packed, sc, gs = nvfp4.pack(w, ld_scale=32)
    dec = nvfp4.decode(packed, sc, gs, N, K, 32)
    # re-quantising the decoded values with the same scales reproduces the codes
    s = np.repeat(nvfp4.E4M3_TABLE[sc[:, : K // 16]], 16, axis=1)
    step = (s * float(gs)).astype(np.float32)
    live = step > 0
    v = np.zeros_like(dec, dtype=np.float32)
    v[live] = (dec[live] / step[live]).astype(np.float32)
    again = nvfp4.e2m1_rne_sat(v)
    again[~live] = 0
    assert np.array_equal(again, nvfp4.unpack_codes(packed, N, K))
    # per-element error bound: half the local grid gap (or the saturation
    # overshoot) times the block's quantisation step
    grid = nvfp4.E2M1_TABLE[:8]
    a = np.abs(w.astype(np.float64)) / np.where(live, step, 1.0)
    idx = np.clip(np.searchsorted(grid, np.minimum(a, 6.0)), 1, 7)
    half_gap = (grid[idx] - grid[idx - 1]) / 2
    bound = np.where(a > 6.0, a - 6.0 + 1e-12, half_gap) * step
    err = np.abs(dec - w.astype(np.float64))
    # w / step is rounded to fp32 before the grid choice: allow one fp32 ulp of it
    slack = np.abs(w.astype(np.float64)) * 2.0 ** -23
    assert np.all(err[live] <= bound[live] + slack[live])
    # blocks whose scale decoded to zero hold only tiny values
    assert np.all(np.abs(w[~live]) <= 6 * float(gs) * 2.0 ** -10 + 1e-30)


def test_pack_scale_is_nearest_e4m3_brute_force():
    g = np.random.default_rng(5)
    w = (g.standard_normal((16, 128)) * 0.02).astype(np.float32)
    _, sc, gs = nvfp4.pack(w)
    denom = np.float32(np.float32(6.0) * gs)
    amax_b = np.abs(w).reshape(16, 8, 16).max(axis=2)
    grid = nvfp4.E4M3_TABLE[:127]
    for n in range(16):
        for b in range(8):
            r = float(np.float32(amax_b[n, b] / denom))
            assert sc[n, b] == _brute_nearest(min(r, 448.0), grid)


def test_decode_rejects_nan_scale():
    with pytest.raises(ValueError):
        nvfp4.decode(np.zeros((1, 8), np.uint8), np.full((1, 1), 0x7F, np.uint8), 1.0, 1, 16, 1)
