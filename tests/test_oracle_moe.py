"""Pins for the oracle's MoE layer (route, permute, expert FFN, combine).

Each check compares the oracle with something other than itself: hand-worked
fixtures, exhaustive search over expert subsets, naive recounts of the
permutation, torch's dense fp64 SwiGLU for the one-expert case, closed forms
and exact invariants of the layer.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from moe_expert_layer_renorm_b200 import inputs
from oracle import moe_layer as M
from oracle import nvfp4
from tests.conftest import golden_lines


# ------------------------------------------------------------------ route ---

def test_route_hand_worked_cases():
    for row in golden_lines("route_worked.txt"):
        assert row[0] == "case"
        bar1 = row.index("|")
        bar2 = row.index("|", bar1 + 1)
        k, E = int(row[1]), int(row[2])
        logits = np.array([[float(v) for v in row[3:bar1]]], np.float32)
        assert logits.shape == (1, E)
        ids_exp = [int(v) for v in row[bar1 + 1:bar2]]
        w_exp = [float(v) for v in row[bar2 + 1:]]
        ids, w = M.route(logits, k)
        assert ids[0].tolist() == ids_exp
        assert np.allclose(w[0], w_exp, rtol=0, atol=1e-7)


def test_route_brute_force_over_subsets():
    E, T = 7, 200
    for k in (1, 2, 3, 7):
        lg = inputs.make_logits(T, E, k, 1.0, seed=42 + k)
        ids, w = M.route(lg, k)
        for t in range(T):
            best = max(itertools.combinations(range(E), k),
                       key=lambda S: sum(float(lg[t, e]) for e in S))
            assert set(ids[t].tolist()) == set(best)
            vals = lg[t, ids[t]]
            assert np.all(np.diff(vals) <= 0)           # descending
            assert abs(w[t].sum() - 1.0) < 1e-12
            assert np.all(np.diff(w[t]) <= 1e-15)


def test_route_modes_agree():
    lg = inputs.make_logits(300, 32, 4, 1.5, seed=9)
    ids, w = M.route(lg, 4)
    w2 = M.softmax_then_renorm(lg, ids)
    assert np.allclose(w, w2, rtol=1e-12, atol=0)


def test_route_tie_goes_to_lower_id():
    lg = np.array([[1.0, 3.0, 3.0, 3.0, 0.0]], np.float32)
    ids, w = M.route(lg, 2)
    assert ids[0].tolist() == [1, 2]


# ---------------------------------------------------------------- permute ---

def test_permute_hand_worked():
    rows = {r[0]: [int(v) for v in r[1:]] for r in golden_lines("permute_worked.txt")}
    ids = np.array(rows["ids"], np.int32).reshape(3, 2)
    off, ps, p2r = M.permute(ids, 3)
    assert off.tolist() == rows["offsets"]
    assert ps.tolist() == rows["perm_src"]
    assert p2r.tolist() == rows["pair_to_row"]


@pytest.mark.parametrize("T,E,k", [(1, 128, 8), (97, 16, 4), (500, 512, 10), (64, 8, 8)])
def test_permute_invariants(T, E, k):
    lg = inputs.make_logits(T, E, k, 1.0, seed=T + E)
    ids, _ = M.route(lg, k)
    off, ps, p2r = M.permute(ids, E)
    flat = ids.reshape(-1)
    naive = [sum(1 for e in flat if e == x) for x in range(E)]
    assert off[0] == 0 and off[-1] == T * k
    assert np.diff(off).tolist() == naive
    assert sorted(ps.tolist()) == list(range(T * k))            # bijection
    for e in range(E):
        grp = ps[off[e]:off[e + 1]]
        assert np.all(flat[grp] == e)
        assert np.all(np.diff(grp) > 0)                          # ascending pair index
    assert np.array_equal(p2r[ps], np.arange(T * k))


# ----------------------------------------------------------------- expert ---

def _nv(codes, scales, g, N, K):
    return M.Nvfp4Tensor(codes, scales, float(np.float32(g)), N, K)


def _packed_expert(H, I, seed, e):
    mats = []
    for which, (N, K) in enumerate(((I, H), (I, H), (H, I))):
        w = inputs.make_weight_fp32_host(N, K, seed, e, which)
        c, s, g = nvfp4.pack(w)
        mats.append(_nv(c, s, g, N, K))
    return M.Expert(*mats)


def _diag(n, code, scale_byte, g):
    """n x n NVFP4 tensor with one E2M1 code on the diagonal, zero elsewhere."""
    q = np.zeros((n, n), np.uint8)
    np.fill_diagonal(q, code)
    packed = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8)
    return _nv(packed, np.full((n, n // 16), scale_byte, np.uint8), g, n, n)


def test_expert_closed_form_diagonal_weights():
    # Wg = a*Id, Wu = b*Id, Wd = c*Id exactly (code 2 = 1.0, scale 0x38 = 1.0):
    # o = c * silu(a x) * (b x) elementwise.
    n = 32
    a, b, c = 0.75, -1.5, 2.0
    ex = M.Expert(_diag(n, 2, 0x38, a), _diag(n, 2, 0x38, b), _diag(n, 2, 0x38, c))
    x = np.linspace(-4, 4, n)[None, :]
    o = M.expert_ffn(x, ex)
    for i in range(n):
        xi = float(x[0, i])
        expect = c * (a * xi / (1.0 + math.exp(-a * xi))) * (b * xi)
        assert abs(o[0, i] - expect) <= 1e-13 * max(1.0, abs(expect))


def test_one_expert_top1_equals_torch_dense_swiglu():
    H, I, T = 64, 96, 24
    ex = _packed_expert(H, I, seed=77, e=0)
    x_bits = inputs.make_x_bits(T, H, seed=78)
    logits = np.zeros((T, 1), np.float32)
    res = M.moe_layer(x_bits, logits, 1, {0: ex})
    xt = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    wg, wu, wd = (torch.from_numpy(t.dense()) for t in (ex.gate, ex.up, ex.down))
    ref = F.linear(F.silu(F.linear(xt, wg)) * F.linear(xt, wu), wd).numpy()
    assert np.allclose(res.y, ref, rtol=1e-12, atol=1e-15)
    assert np.array_equal(res.ids, np.zeros((T, 1), np.int32))
    assert np.allclose(res.w, 1.0)


def test_all_experts_selected_is_a_dense_mixture():
    # k = E: every expert sees every token and y = sum_e softmax(l)_e * FFN_e(x)
    H, I, T, E = 32, 48, 10, 4
    exps = {e: _packed_expert(H, I, seed=5, e=e) for e in range(E)}
    x_bits = inputs.make_x_bits(T, H, seed=6)
    lg = inputs.make_logits(T, E, E, 1.0, seed=7)
    res = M.moe_layer(x_bits, lg, E, exps)
    xt = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    p = torch.softmax(torch.from_numpy(lg).to(torch.float64), dim=1)
    ref = torch.zeros(T, H, dtype=torch.float64)
    for e, ex in exps.items():
        wg, wu, wd = (torch.from_numpy(t.dense()) for t in (ex.gate, ex.up, ex.down))
        ref += p[:, e:e + 1] * F.linear(F.silu(F.linear(xt, wg)) * F.linear(xt, wu), wd)
    assert np.allclose(res.y, ref.numpy(), rtol=1e-11, atol=1e-14)


def test_identical_experts_make_routing_irrelevant():
    H, I, T, E, k = 32, 32, 12, 6, 3
    ex = _packed_expert(H, I, seed=8, e=0)
    x_bits = inputs.make_x_bits(T, H, seed=9)
    lg = inputs.make_logits(T, E, k, 1.0, seed=10)
    res = M.moe_layer(x_bits, lg, k, {e: ex for e in range(E)})
    single = M.expert_ffn(M.bf16_bits_to_f64(x_bits), ex)
    assert np.allclose(res.y, single, rtol=1e-12, atol=1e-15)


def test_down_global_scale_doubles_output_exactly():
    H, I, T, E, k = 32, 64, 9, 4, 2
    exps = {e: _packed_expert(H, I, seed=11, e=e) for e in range(E)}
    x_bits = inputs.make_x_bits(T, H, seed=12)
    lg = inputs.make_logits(T, E, k, 1.0, seed=13)
    y1 = M.moe_layer(x_bits, lg, k, exps).y
    doubled = {e: M.Expert(ex.gate, ex.up, M.Nvfp4Tensor(ex.down.codes, ex.down.scales,
                                                         2 * ex.down.global_scale, H, I))
               for e, ex in exps.items()}
    y2 = M.moe_layer(x_bits, lg, k, doubled).y
    assert np.array_equal(y2, 2 * y1)


def test_relabelling_experts_leaves_output_unchanged():
    H, I, T, E, k = 32, 32, 15, 5, 2
    exps = {e: _packed_expert(H, I, seed=14, e=e) for e in range(E)}
    x_bits = inputs.make_x_bits(T, H, seed=15)
    lg = inputs.make_logits(T, E, k, 1.0, seed=16)
    perm = np.array([3, 0, 4, 1, 2])                # new id of old expert e is perm[e]
    lg2 = np.empty_like(lg)
    lg2[:, perm] = lg
    exps2 = {int(perm[e]): ex for e, ex in exps.items()}
    # pairs are ordered by (token, rank), so y does not depend on the labels
    y1 = M.moe_layer(x_bits, lg, k, exps).y
    y2 = M.moe_layer(x_bits, lg2, k, exps2).y
    assert np.allclose(y1, y2, rtol=1e-13, atol=1e-16)


def test_sampled_tokens_match_full_layer():
    H, I, T, E, k = 32, 32, 40, 8, 2
    exps = {e: _packed_expert(H, I, seed=17, e=e) for e in range(E)}
    x_bits = inputs.make_x_bits(T, H, seed=18)
    lg = inputs.make_logits(T, E, k, 1.0, seed=19)
    full = M.moe_layer(x_bits, lg, k, exps)
    toks = [0, 7, 39, 13]
    part = M.moe_layer(x_bits, lg, k, exps, tokens=toks)
    assert np.allclose(part.y, full.y[toks], rtol=1e-13, atol=1e-16)
    # out_perm rows recombine to y
    o = full.out_perm[full.pair_to_row].reshape(T, k, H)
    assert np.allclose((o * full.w[:, :, None]).sum(axis=1), full.y, rtol=1e-13, atol=1e-16)


def test_tolerance_formula():
    y = np.array([[3.0, -4.0]])                      # rms = sqrt(12.5)
    assert abs(M.tolerance(y) - (1e-2 * math.sqrt(12.5) + 1e-3)) < 1e-15
