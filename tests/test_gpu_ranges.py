"""The layer across the range of activation magnitudes that bf16 can hold.

The kernels multiply f16 operands: each token row is brought to a largest
magnitude in [2^14, 2^15) by a power of two before its f16 conversion, and h
is stored normalised by the square of the row's factor (see the header's
ft_moe_ffn_nvfp4).  These tests scale whole token rows by powers of two far
from 1 and check every output row against the oracle at a bound RELATIVE to
that row (the layer tolerance's absolute floor would hide an error on rows
of small magnitude), on both expert kernels; and they drive h past the f16
range on purpose to check that the overflow is reported, not silent."""
import dataclasses

import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.layer import ExpertPool, MoELayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS

# decode kernel: a few rows per expert; prefill (tcgen05) kernels: 100 rows per expert, and 400 (the
# gate/up GEMM's large-group shape, A in shared memory)
SHAPES = {
    "decode": inputs.custom_workload(W["tiny"], T=40, seed=5151),
    "prefill": inputs.custom_workload(W["tiny"], H=256, I=256, E=4, k=4, T=100, seed=5152),
    "prefill_large": inputs.custom_workload(W["tiny"], H=256, I=256, E=4, k=4, T=400, seed=5153),
}


def scale_rows(x_bits: np.ndarray, exps) -> np.ndarray:
    """bf16 rows times 2^exps[t] (exact: a power of two moves only the exponent)."""
    x = (x_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    x = x * np.exp2(np.asarray(exps, np.float64))[:, None]
    out = (x.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    back = (out.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(back.astype(np.float64), x), "scaling left the bf16 normal range"
    return out


def check_rows_relative(run, k, rel=1e-2):
    T = run.x_bits.shape[0]
    ref = G.reference_y(run, k, np.arange(T))
    for t in range(T):
        rms = float(np.sqrt(np.mean(ref[t] ** 2)))
        err = float(np.abs(run.y[t] - ref[t]).max())
        assert rms > 0 and err <= rel * rms, f"row {t}: max |err| {err:.3g} > {rel} * rms {rms:.3g}"


@pytest.mark.parametrize("kernel", sorted(SHAPES))
@pytest.mark.parametrize("exp", [20, -20])
def test_uniformly_scaled_rows(cuda_device, kernel, exp):
    w = SHAPES[kernel]
    li = inputs.make_layer_inputs(w)
    li = dataclasses.replace(li, x_bits=scale_rows(li.x_bits, [exp] * w.T))
    run = G.run_gpu(w, li=li)
    G.check_routing(run, w.k)
    check_rows_relative(run, w.k)


@pytest.mark.parametrize("kernel", sorted(SHAPES))
def test_rows_of_mixed_magnitude(cuda_device, kernel):
    # one batch holding rows at 2^-30, 2^-20, 1, 2^20 and 2^30
    w = SHAPES[kernel]
    li = inputs.make_layer_inputs(w)
    exps = [(-30, -20, 0, 20, 30)[t % 5] for t in range(w.T)]
    li = dataclasses.replace(li, x_bits=scale_rows(li.x_bits, exps))
    run = G.run_gpu(w, li=li)
    G.check_routing(run, w.k)
    check_rows_relative(run, w.k)


def _constant_pool(w, value: float):
    pool = ExpertPool(w.H, w.I, w.E)
    for e in range(w.E):
        for mat in range(3):
            N, K = pool.shape(mat)
            pool.pack_into(e, mat, torch.full((N, K), value, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    return pool, np.arange(w.E, dtype=np.int32)


def _constant_rows(w, value: float) -> inputs.LayerInputs:
    li = inputs.make_layer_inputs(w)
    bits = np.full_like(li.x_bits, np.frombuffer(np.float32(value).tobytes(), np.uint32)[0] >> 16)
    return dataclasses.replace(li, x_bits=bits)


@pytest.mark.parametrize("kernel", sorted(SHAPES))
def test_h_beyond_f16_range_is_reported(cuda_device, kernel):
    # every weight 1 and every activation 4: gate and up are 4 H = 1024 for every feature, so
    # h = silu(1024) * 1024 ~ 1.05e6, beyond the f16 maximum 65504: the kernels saturate and
    # record FT_DEV_F16_RANGE
    w = SHAPES[kernel]
    pool, st = _constant_pool(w, 1.0)
    G.run_gpu(w, pool=pool, slot_table=st, li=_constant_rows(w, 4.0), expect_status=_lib.FT_DEV_F16_RANGE)
    assert _lib.device_status(clear=True) == _lib.FT_DEV_OK   # the word was read and cleared


@pytest.mark.parametrize("kernel", sorted(SHAPES))
def test_h_near_f16_limit_is_exact_enough(cuda_device, kernel):
    # weights 1/8 and activations 4: gate and up are H / 2 = 128, h = silu(128) * 128 = 16384,
    # inside the f16 range: no status, and the outputs match the oracle row by row
    w = SHAPES[kernel]
    pool, st = _constant_pool(w, 0.125)
    run = G.run_gpu(w, pool=pool, slot_table=st, li=_constant_rows(w, 4.0))
    check_rows_relative(run, w.k)
