"""Pins of the oracle's MXFP4 format: E2M1 elements sharing one E8M0 scale
per 32 values, the format the pages list beside NVFP4 ("FlashML-org /
FreeToken" about page, quantization formats; model guide, CPU executor
formats).  The pages define neither the format nor a conversion, so the
oracle follows the OCP Microscaling Formats (MX) v1.0 specification; these
tests pin it by closed forms, a hand-worked example, brute force and exact
invariants, not by retyping its code."""
import math

import numpy as np
import pytest

from oracle import cpp

# E2M1 magnitudes by the 3 low code bits (bit 3 is the sign): hand table
E2M1_MAG = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _nibbles(codes: np.ndarray, K: int) -> np.ndarray:
    out = np.empty((codes.shape[0], K), np.int64)
    out[:, 0::2] = codes & 15
    out[:, 1::2] = codes >> 4
    return out


def test_e8m0_closed_form():
    for b in range(255):
        assert cpp.e8m0_value(b) == math.ldexp(1.0, b - 127)
    assert math.isnan(cpp.e8m0_value(255))


def test_hand_worked_blocks():
    w = np.zeros((1, 128), np.float32)
    # block 0: amax 7, floor(log2 7) = 2, shared exponent 2 - 2 = 0, scale 2^0 (byte 127)
    #   6 -> 6 (code 7); 3 -> code 5; -1.5 -> 8 | 3 = 11; 0.25: tie of 0 and 0.5 -> even index 0;
    #   0.75: tie of 0.5 (index 1) and 1.0 (index 2) -> even index 2 (code 2);
    #   -0.0 -> code 8; 5: tie of 4 (index 6) and 6 (index 7) -> index 6 (code 6); 7 saturates to 6 (code 7)
    w[0, :8] = [6.0, 3.0, -1.5, 0.25, 0.75, -0.0, 5.0, 7.0]
    # block 1: amax 0.8, floor(log2 0.8) = -1, shared exponent -3, scale 1/8 (byte 124)
    #   0.8 * 8 = 6.4 saturates to 6 (code 7); 0.1 * 8 = 0.8 -> 1 (code 2);
    #   -0.05 * 8 = -0.4 -> -0.5 (code 9); 0.3 * 8 = 2.4 -> 2 (code 4)
    w[0, 32:36] = [0.8, 0.1, -0.05, 0.3]
    # block 2: all zero -> the smallest scale (byte 0), codes 0
    # block 3: amax 2^-130: floor(log2) - 2 = -132 is clamped to -127 (byte 0);
    #   2^-130 / 2^-127 = 1/8 rounds to 0
    w[0, 96] = np.float32(2.0 ** -130)
    codes, scales = cpp.pack_mxfp4(w)
    assert scales.tolist() == [[127, 124, 0, 0]]
    c = _nibbles(codes, 128)[0]
    assert c[:8].tolist() == [7, 5, 11, 0, 2, 8, 6, 7]
    assert c[8:32].tolist() == [0] * 24
    assert c[32:36].tolist() == [7, 2, 9, 4]
    assert not c[36:].any()
    v = cpp.decode_mxfp4(codes, scales, 128)[0]
    assert v[:8].tolist() == [6.0, 3.0, -1.5, 0.0, 1.0, 0.0, 4.0, 6.0]
    assert math.copysign(1.0, v[5]) == -1.0
    assert v[32:36].tolist() == [0.75, 0.125, -0.0625, 0.25]


def test_power_of_two_scaling_moves_only_the_scale():
    w = (np.random.default_rng(3).standard_normal((4, 256)) * 0.02).astype(np.float32)
    c0, s0 = cpp.pack_mxfp4(w)
    for j in (-9, 1, 24):
        c1, s1 = cpp.pack_mxfp4((w * np.float32(2.0 ** j)).astype(np.float32))
        assert np.array_equal(c1, c0)
        assert np.array_equal(s1.astype(np.int64), s0.astype(np.int64) + j)


def test_scale_brackets_the_block_maximum():
    w = (np.random.default_rng(5).standard_normal((8, 512)) * np.float32(0.3)).astype(np.float32)
    _, s = cpp.pack_mxfp4(w)
    blocks = np.abs(w.astype(np.float64)).reshape(8, 16, 32).max(axis=2)
    ratio = blocks / np.ldexp(1.0, s.astype(np.int64) - 127)
    assert ((ratio >= 4.0) & (ratio < 8.0)).all()   # the largest element lands in E2M1's top binade


def test_codes_are_the_nearest_values_given_the_scale():
    """Brute force over all 16 codes: the nearest decoded value, ties to the
    even magnitude index, above 6 the largest, and the sign of w kept."""
    rng = np.random.default_rng(7)
    w = (rng.standard_normal((6, 64)) * np.float32(0.05)).astype(np.float32)
    w[0, :4] = [0.0, -0.0, 1e-30, -1e-30]
    codes, scales = cpp.pack_mxfp4(w)
    c = _nibbles(codes, 64)
    for n in range(6):
        for k in range(64):
            x = float(w[n, k])
            X = math.ldexp(1.0, int(scales[n, k // 32]) - 127)
            a = abs(x) / X
            best = min(range(8), key=lambda i: (abs(E2M1_MAG[i] - a), i % 2))
            if a > 6.0:
                best = 7
            sign = 8 if math.copysign(1.0, x) < 0 else 0
            assert c[n, k] == best | sign, (n, k, x)


def test_representable_blocks_round_trip():
    rng = np.random.default_rng(11)
    N, K = 5, 256
    codes_n = rng.integers(0, 16, size=(N, K))
    codes_n[:, ::32] = rng.choice([6, 7, 14, 15], size=(N, K // 32))   # each block reaches 4 or 6
    sc = rng.integers(100, 150, size=(N, K // 32)).astype(np.uint8)
    vals = np.array([math.copysign(E2M1_MAG[c & 7], -1.0 if c & 8 else 1.0) for c in codes_n.ravel()])
    vals = vals.reshape(N, K) * np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=1))
    codes, scales = cpp.pack_mxfp4(vals.astype(np.float32))
    assert np.array_equal(scales, sc)
    assert np.array_equal(_nibbles(codes, K), codes_n)
    assert np.array_equal(cpp.decode_mxfp4(codes, scales, K), vals)


def test_rejects_bad_inputs():
    with pytest.raises(ValueError):
        cpp.pack_mxfp4(np.zeros((2, 48), np.float32))
    bad = np.zeros((1, 32), np.float32)
    bad[0, 3] = np.nan
    with pytest.raises(ValueError):
        cpp.pack_mxfp4(bad)
    with pytest.raises(ValueError):
        cpp.decode_mxfp4(np.zeros((1, 16), np.uint8), np.full((1, 1), 255, np.uint8), 32)


def test_numpy_and_cpp_oracles_agree_bit_for_bit():
    """Two MXFP4 implementations written apart (numpy, C++) on random,
    scaled, tied and saturating inputs."""
    from oracle import mxfp4
    g = np.random.default_rng(13)
    w = (g.standard_normal((6, 128)) * np.float32(0.04)).astype(np.float32)
    w[1] *= np.float32(2.0 ** 40)
    w[2] *= np.float32(2.0 ** -60)
    w[3, :8] = [0.25, 0.75, 5.0, 7.0, -0.0, 1e-30, -6.5, 2.5]
    w[4, 32:64] = 0.0
    c1, s1 = cpp.pack_mxfp4(w)
    c2, s2 = mxfp4.pack(w)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    assert np.array_equal(cpp.decode_mxfp4(c1, s1, 128), mxfp4.decode(c2, s2, 128))


def test_layer_with_mxfp4_experts_is_the_dense_layer():
    """The oracle's layer over MXFP4 experts read from a slot pool (each E8M0
    byte stored at both of its 16-K positions, the global ignored) equals the
    same layer computed densely from decode_mxfp4 of each tensor."""
    import bench
    from moe_expert_layer_renorm_b200 import inputs
    w = inputs.WORKLOADS["tiny"]
    L = bench.reference_layout(w.H, w.I)
    s = inputs.layer_seed(w.seed, 0)
    st = np.arange(w.E, dtype=np.int32)
    pool = np.zeros(w.E * L["slot_bytes"], np.uint8)
    dense = {}
    shapes = [(w.I, w.H), (w.I, w.H), (w.H, w.I)]
    for e in range(w.E):
        base = e * L["slot_bytes"]
        mats = []
        for m, (N, K) in enumerate(shapes):
            wt = inputs.make_weight_fp32_host(N, K, s, e, m)
            codes, sc = cpp.pack_mxfp4(wt)
            mats.append(cpp.decode_mxfp4(codes, sc, K))
            ld = L["ld_scale"][m]
            sc16 = np.zeros((N, ld), np.uint8)
            sc16[:, 0:K // 16:2] = sc
            sc16[:, 1:K // 16:2] = sc
            o = base + L["codes_off"][m]
            pool[o:o + codes.size] = codes.reshape(-1)
            o = base + L["scales_off"][m]
            pool[o:o + sc16.size] = sc16.reshape(-1)
            o = base + L["global_off"][m]
            pool[o:o + 4] = np.frombuffer(np.float32(1024.0).tobytes(), np.uint8)   # must not matter
        dense[e] = mats
    li = inputs.make_layer_inputs(w)
    y = cpp.moe_layer(li.x_bits, li.logits, w.k, st, pool, L["slot_bytes"], L["codes_off"], L["scales_off"],
                      L["global_off"], L["ld_scale"], w.H, w.I, fmt=1)
    ids, wts = cpp.route(li.logits, w.k)
    x = inputs.bf16_bits_to_fp32(li.x_bits).astype(np.float64)
    ref = np.zeros_like(y)
    for t in range(x.shape[0]):
        for j in range(w.k):
            g_, u_, d_ = dense[int(ids[t, j])]
            G, U = g_ @ x[t], u_ @ x[t]
            ref[t] += wts[t, j] * (d_ @ (G * U / (1.0 + np.exp(-G))))
    assert np.max(np.abs(y - ref)) <= 1e-12 * np.max(np.abs(ref))
