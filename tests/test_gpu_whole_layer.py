"""ft_moe_layer_nvfp4, the whole layer as one call, against the four separate
calls (ft_moe_route, ft_moe_permute, ft_moe_ffn_nvfp4, ft_moe_combine) on the
same inputs: every output -- ids, weights, offsets, both permutations, the
expert outputs and y -- must be identical bit for bit, on decode-sized
batches (one persistent launch) and on larger ones (the four calls inside).
Also: repeated calls and a call that records a device status leave the
workspace ready for the next call; graph capture; both scale formats and
both slot arrangements.  Parity with the oracle itself is covered by the
layer tests, which go through this call."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.layer import MoELayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS

OUTPUTS = ("ids", "w", "offsets", "perm_src", "pair_to_row", "out_perm", "y")


def _tensors(w, li, slot_table):
    x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    lg = torch.from_numpy(li.logits).cuda()
    st = torch.from_numpy(np.asarray(slot_table, dtype=np.int32)).cuda()
    return x, lg, st


def _run(w, li, pool, st_host, whole: bool):
    x, lg, st = _tensors(w, li, st_host)
    lay = MoELayer(li.x_bits.shape[0], w.E, w.k, w.H, w.I, mode=w.route_mode, whole=whole)
    G.poison(lay)
    _lib.device_status(clear=True)
    lay.forward(x, lg, st, pool)
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == _lib.FT_DEV_OK
    return lay


def _assert_same(a: MoELayer, b: MoELayer):
    for name in OUTPUTS:
        ta, tb = getattr(a, name), getattr(b, name)
        assert torch.equal(ta.view(torch.int32) if ta.dtype == torch.float32 else ta,
                           tb.view(torch.int32) if tb.dtype == torch.float32 else tb), name


CASES = {
    "tiny": W["tiny"],
    "decode_T1": W["decode_T1"],
    "decode_T8": W["decode_T8"],
    "decode_T64": W["decode_T64"],
    "slots512_T1": W["slots512_T1"],
    "wide_decode_T1": W["wide_decode_T1"],
    # K not a multiple of 256, features not a multiple of 128, ragged groups
    "ragged_320x448": inputs.custom_workload(W["tiny"], H=320, I=448, E=8, k=2, T=40, seed=4562),
    # 128 tokens, 1024 pairs (the most one launch takes), and 96 tokens over 512 experts
    "T128": inputs.custom_workload(W["decode_T64"], T=128, seed=4563),
    "T96_E512": inputs.custom_workload(W["slots512_T1"], T=96, seed=4565),
    # larger batches: the four calls run inside the one call
    "prefill_small": inputs.custom_workload(W["tiny"], H=256, I=256, E=4, k=4, T=100, seed=4564),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_whole_layer_equals_the_four_calls(cuda_device, name):
    w = CASES[name]
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w)
    a = _run(w, li, pool, st, whole=True)
    b = _run(w, li, pool, st, whole=False)
    _assert_same(a, b)
    assert not torch.isnan(a.y).any()


def test_whole_layer_matches_the_oracle_at_its_limits(cuda_device):
    w = CASES["T128"]
    run = G.run_gpu(w, whole=True)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)


def test_calls_leave_the_workspace_ready(cuda_device):
    # the same layer object (one workspace) called again and again, with a call that records a
    # device status (a non-resident expert) in between: every clean call gives the same bits
    w = W["decode_T8"]
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w)
    x, lg, stt = _tensors(w, li, st)
    lay = MoELayer(w.T, w.E, w.k, w.H, w.I, mode=w.route_mode, whole=True)
    _lib.device_status(clear=True)
    lay.forward(x, lg, stt, pool)
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == _lib.FT_DEV_OK
    first = {n: getattr(lay, n).clone() for n in OUTPUTS}
    ids, _ = G.M.route(li.logits, w.k)
    bad = stt.clone()
    bad[int(ids[0, 0])] = -1
    for i in range(4):
        lay.forward(x, lg, bad if i == 2 else stt, pool)
        torch.cuda.synchronize()
        status = _lib.device_status(clear=True)
        if i == 2:
            assert status == _lib.FT_DEV_NOT_RESIDENT
            continue
        assert status == _lib.FT_DEV_OK
        for n in OUTPUTS:
            assert torch.equal(getattr(lay, n), first[n]), (i, n)


def test_whole_layer_in_a_cuda_graph(cuda_device):
    w = W["decode_T32"]
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w)
    x, lg, stt = _tensors(w, li, st)
    lay = MoELayer(w.T, w.E, w.k, w.H, w.I, mode=w.route_mode, whole=True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        lay.forward(x, lg, stt, pool, stream=s)
        torch.cuda.synchronize()
        ref = lay.y.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            lay.forward(x, lg, stt, pool, stream=s)
    for _ in range(3):
        lay.y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(lay.y, ref)
    g.reset()


@pytest.mark.parametrize("fmt,tiled", [(_lib.FT_SCALE_MXFP4, False), (_lib.FT_SCALE_NVFP4, True)])
def test_whole_layer_formats_and_slot_layouts(cuda_device, fmt, tiled):
    w = W["decode_T8"]
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w, fmt=fmt, tiled=tiled)
    a = _run(w, li, pool, st, whole=True)
    b = _run(w, li, pool, st, whole=False)
    _assert_same(a, b)
