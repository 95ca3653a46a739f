"""Pins for the C++ oracle (oracle/moe_oracle.cpp).

The C++ oracle is written apart from the numpy oracle; it is pinned here to
the same hand-worked fixtures, closed forms and invariants, to brute force on
tiny inputs, and bit for bit (indexing, packing) or to fp64 rounding (the
layer) to the numpy oracle on random inputs of every workload family.
"""
import itertools

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from moe_expert_layer_renorm_b200 import inputs
from oracle import cpp as C
from oracle import moe_layer as M
from oracle import nvfp4
from tests.conftest import golden_lines


# ----------------------------------------------------------------- decode ---

def test_e2m1_codes_hand_worked():
    rows = golden_lines("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        v = C.e2m1_value(int(code))
        assert v == float(val) and np.signbit(v) == val.startswith("-")


def test_e4m3_spot_values_hand_worked():
    for byte, val in golden_lines("e4m3_spot.txt"):
        v = C.e4m3_value(int(byte, 16))
        if val.lower() == "nan":
            assert np.isnan(v)
        else:
            assert v == float(val)


def test_e4m3_all_codes_closed_form():
    for b in range(256):
        s, e, m = b >> 7, (b >> 3) & 15, b & 7
        v = C.e4m3_value(b)
        if e == 15 and m == 7:
            assert np.isnan(v)
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        assert v == (-mag if s else mag)


def test_e4m3_all_codes_match_torch_float8():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([C.e4m3_value(b) for b in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


# ------------------------------------------------------------------- pack ---

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
    packed, sc, g = C.pack(w)
    assert float(g) == gexp
    assert np.array_equal(sc, scales)
    unpacked = np.stack([packed & 15, packed >> 4], axis=2).reshape(2, 32)   # even k in the low nibble
    assert np.array_equal(unpacked, codes)


def test_e2m1_rounding_hand_worked_through_pack():
    # a block whose largest magnitude is 6 * 2^-12 * 448 = 6 * 448 g with g = 2^-12
    # has scale 448 and step 448 g; dividing by that step gives back the
    # fixture's inputs, so each rounds to the fixture's code
    checked = 0
    for v, code in golden_lines("e2m1_rounding.txt"):
        if abs(float(v)) > 6.0:
            continue                # would raise the block maximum; the saturation pins cover it
        g = 2.0 ** -12
        step = 448 * g
        w = np.zeros((1, 16), np.float32)
        w[0, 0] = 6 * step          # sets amax = 2688 g, hence the global scale g and scale byte 448
        w[0, 1] = np.float32(float(v) * step)
        if np.float32(w[0, 1]) / np.float32(step) != np.float32(float(v)):
            continue                # not representable after scaling; the numpy pins cover it
        codes, scales, gg = C.pack(w)
        assert float(gg) == g and scales[0, 0] == 0x7E
        assert (codes[0, 0] >> 4) == int(code), v
        checked += 1
    assert checked >= 10


@pytest.mark.parametrize("N,K,seed", [(64, 256, 1), (17, 2880, 2), (3, 16, 3), (128, 2048, 4)])
def test_pack_bit_exact_with_numpy_oracle(N, K, seed):
    g = np.random.default_rng(seed)
    w = (g.standard_normal((N, K)) * 0.02).astype(np.float32)
    w[0, :16] = 0.0                                  # an all-zero block
    w[min(1, N - 1), 16:32] *= 1e-30                 # a block that underflows its scale
    if N > 2:
        w[2, 5] = 7.5                                # one large outlier
    ld = (K // 16 + 15) // 16 * 16
    a = C.pack(w, ld)
    b = nvfp4.pack(w, ld)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2] == b[2]


def test_pack_all_zero_tensor():
    codes, scales, g = C.pack(np.zeros((4, 64), np.float32))
    assert g == 1.0 and not codes.any() and not scales.any()


# ------------------------------------------------------------------ route ---

def test_route_hand_worked_cases():
    for row in golden_lines("route_worked.txt"):
        bar1 = row.index("|")
        bar2 = row.index("|", bar1 + 1)
        k, E = int(row[1]), int(row[2])
        logits = np.array([[float(v) for v in row[3:bar1]]], np.float32)
        ids, w = C.route(logits, k)
        assert ids[0].tolist() == [int(v) for v in row[bar1 + 1:bar2]]
        # the fixture's weights are exact for the written logits; fp32 logits move them by < 1e-7
        assert np.allclose(w[0], [float(v) for v in row[bar2 + 1:]], rtol=0, atol=1e-7)


def test_route_brute_force_over_subsets():
    E, T = 7, 150
    for k in (1, 2, 3, 7):
        lg = inputs.make_logits(T, E, k, 1.0, seed=77 + k)
        ids, w = C.route(lg, k)
        for t in range(T):
            best = max(itertools.combinations(range(E), k), key=lambda S: sum(float(lg[t, e]) for e in S))
            assert set(ids[t].tolist()) == set(best)
            assert np.all(np.diff(lg[t, ids[t]]) <= 0)
            assert abs(w[t].sum() - 1.0) < 1e-12


def test_route_tie_goes_to_lower_id():
    lg = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]], np.float32)
    ids, w = C.route(lg, 2)
    assert ids[0].tolist() == [1, 2] and w[0, 0] == w[0, 1] == 0.5


@pytest.mark.parametrize("T,E,k", [(300, 128, 8), (200, 512, 10), (100, 32, 4), (64, 8, 2)])
def test_route_matches_numpy_oracle(T, E, k):
    lg = inputs.make_logits(T, E, k, 1.0, seed=T + E)
    a, wa = C.route(lg, k)
    b, wb = M.route(lg, k)
    assert np.array_equal(a, b)
    assert np.allclose(wa, wb, rtol=1e-14, atol=0)


# ---------------------------------------------------------------- permute ---

def test_permute_hand_worked():
    rows = {r[0]: [int(v) for v in r[1:]] for r in golden_lines("permute_worked.txt")}
    ids = np.array(rows["ids"], np.int32).reshape(3, 2)
    off, ps, p2r = C.permute(ids, 3)
    assert off.tolist() == rows["offsets"] and ps.tolist() == rows["perm_src"]
    assert p2r.tolist() == rows["pair_to_row"]


@pytest.mark.parametrize("T,E,k", [(1, 128, 8), (333, 32, 4), (2048, 512, 10)])
def test_permute_matches_numpy_oracle(T, E, k):
    g = np.random.default_rng(T * E)
    ids = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    for a, b in zip(C.permute(ids, E), M.permute(ids, E)):
        assert np.array_equal(a, b)


# ------------------------------------------------------------------ layer ---

def _layout(H: int, I: int):
    """The slot layout of the library's C header, as the bench's reference arm
    writes it out (checked against the library in test_abi)."""
    import bench
    return bench.reference_layout(H, I)


def _pool(w: inputs.Workload, layer: int = 0):
    """A host slot pool in the library's layout, packed by the numpy oracle."""
    L = _layout(w.H, w.I)
    s = inputs.layer_seed(w.seed, layer)
    st = inputs.make_slot_table(w.E, w.slots, w.permuted_slots, s)
    pool = np.zeros(w.slots * L["slot_bytes"], np.uint8)
    exps = {}
    shapes = [(w.I, w.H), (w.I, w.H), (w.H, w.I)]
    for e in range(w.E):
        base = int(st[e]) * L["slot_bytes"]
        mats = []
        for m, (N, K) in enumerate(shapes):
            c, sc, g = nvfp4.pack(inputs.make_weight_fp32_host(N, K, s, e, m), L["ld_scale"][m])
            o = base + L["codes_off"][m]
            pool[o:o + c.size] = c.reshape(-1)
            o = base + L["scales_off"][m]
            pool[o:o + sc.size] = sc.reshape(-1)
            o = base + L["global_off"][m]
            pool[o:o + 4] = np.frombuffer(np.float32(g).tobytes(), np.uint8)
            mats.append(M.Nvfp4Tensor(c, sc, g, N, K))
        exps[e] = M.Expert(*mats)
    return L, st, pool, exps


def _cpp_layer(w, li, L, st, pool, tokens=None, k=None):
    return C.moe_layer(li.x_bits, li.logits, k or w.k, st, pool, L["slot_bytes"], L["codes_off"], L["scales_off"],
                       L["global_off"], L["ld_scale"], w.H, w.I, tokens=tokens)


@pytest.mark.parametrize("name", ["tiny"])
def test_layer_matches_numpy_oracle(name):
    w = inputs.WORKLOADS[name]
    L, st, pool, exps = _pool(w)
    li = inputs.make_layer_inputs(w)
    y = _cpp_layer(w, li, L, st, pool)
    ref = M.moe_layer(li.x_bits, li.logits, w.k, exps).y
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_layer_matches_numpy_oracle_sampled_decode_config():
    w = inputs.custom_workload(inputs.WORKLOADS["decode_T8"], E=16, n_slots=None)
    L, st, pool, exps = _pool(w)
    li = inputs.make_layer_inputs(w)
    tok = [0, 5, 7]
    y = _cpp_layer(w, li, L, st, pool, tokens=tok)
    ref = M.moe_layer(li.x_bits, li.logits, w.k, exps, tokens=np.array(tok)).y
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_one_expert_top1_equals_torch_dense_swiglu():
    w = inputs.custom_workload(inputs.WORKLOADS["tiny"], E=1, k=1, T=6)
    L, st, pool, exps = _pool(w)
    li = inputs.make_layer_inputs(w)
    y = _cpp_layer(w, li, L, st, pool)
    ex = exps[0]
    x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    wg, wu, wd = (torch.from_numpy(t.dense()) for t in (ex.gate, ex.up, ex.down))
    ref = F.linear(F.silu(F.linear(x, wg)) * F.linear(x, wu), wd)
    assert np.max(np.abs(y - ref.numpy())) <= 1e-12 * float(ref.abs().max())


def test_identical_experts_make_routing_irrelevant():
    # every expert id maps to the same slot, so each token's output is that
    # expert's output times the sum of its combine weights, which is 1
    import dataclasses
    w = inputs.custom_workload(inputs.WORKLOADS["tiny"], T=5)
    L, st, pool, exps = _pool(w)
    li = inputs.make_layer_inputs(w)
    same = np.full_like(st, st[0])
    y_all = _cpp_layer(w, li, L, same, pool)
    one = dataclasses.replace(li, logits=np.ascontiguousarray(li.logits[:, :1]))
    y_one = C.moe_layer(one.x_bits, one.logits, 1, same[:1], pool, L["slot_bytes"], L["codes_off"],
                        L["scales_off"], L["global_off"], L["ld_scale"], w.H, w.I)
    assert np.max(np.abs(y_all - y_one)) <= 1e-12 * np.max(np.abs(y_one))


def test_non_resident_expert_is_an_error():
    w = inputs.WORKLOADS["tiny"]
    L, st, pool, _ = _pool(w)
    li = inputs.make_layer_inputs(w)
    bad = st.copy()
    bad[:] = -1
    with pytest.raises(ValueError, match="not resident"):
        _cpp_layer(w, li, L, bad, pool, tokens=[0])
