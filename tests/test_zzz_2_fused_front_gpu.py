"""ft_moe_route_permute (route and permute in one launch for small batches)
against the two calls it replaces, bit for bit, and against the oracle's
routing and permutation; then a whole layer through it against the oracle.

Collected after the rest of the GPU suite, before the expert-parallel tests."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from oracle import moe_layer as M
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _logits(T, E, k, seed, ties):
    g = np.random.default_rng(seed)
    if ties:   # small integers: many equal logits, so the lower-id rule decides
        return g.integers(-3, 4, size=(T, E)).astype(np.float32)
    return inputs.make_logits(T, E, k, 1.0, seed)


def _buffers(T, E, k):
    P = max(T * k, 1)
    dev = "cuda"
    return dict(ids=torch.full((P,), -7, dtype=torch.int32, device=dev),
                w=torch.full((P,), float("nan"), dtype=torch.float32, device=dev),
                off=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
                ps=torch.full((P,), -7, dtype=torch.int32, device=dev),
                p2r=torch.full((P,), -7, dtype=torch.int32, device=dev))


# fused sizes (T <= 128, T*k <= 1024, E <= 512) and sizes that take the two-call path
SHAPES = [(1, 128, 8), (8, 128, 8), (64, 128, 8), (128, 128, 8), (16, 8, 2), (128, 8, 8), (1, 512, 10),
          (100, 512, 10), (33, 32, 4), (5, 1, 1), (128, 64, 8), (7, 33, 32),
          (129, 128, 8), (256, 128, 8), (64, 1024, 8), (64, 600, 4)]


@pytest.mark.parametrize("T,E,k", SHAPES)
@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("ties", [False, True])
def test_route_permute_equals_the_two_calls(cuda_device, T, E, k, mode, ties):
    lg = _logits(T, E, k, seed=T * 7919 + E * 31 + k + mode, ties=ties)
    d_lg = torch.from_numpy(lg).cuda()
    wsb = _lib.permute_workspace_size(T, k, E)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
    a, b = _buffers(T, E, k), _buffers(T, E, k)
    _lib.device_status(clear=True)
    s = _stream()
    _lib.route(d_lg.data_ptr(), T, E, k, mode, a["ids"].data_ptr(), a["w"].data_ptr(), s)
    _lib.permute(a["ids"].data_ptr(), T, k, E, a["off"].data_ptr(), a["ps"].data_ptr(), a["p2r"].data_ptr(),
                 ws.data_ptr(), wsb, s)
    _lib.route_permute(d_lg.data_ptr(), T, E, k, mode, b["ids"].data_ptr(), b["w"].data_ptr(), b["off"].data_ptr(),
                       b["ps"].data_ptr(), b["p2r"].data_ptr(), ws.data_ptr(), wsb, s)
    torch.cuda.synchronize()
    assert _lib.device_status(clear=True) == 0
    for key in ("ids", "off", "ps", "p2r"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["w"].view(torch.int32), b["w"].view(torch.int32))     # the same bits
    ids, _ = M.route(lg, k)
    off, ps, p2r = M.permute(ids, E)
    assert np.array_equal(b["ids"].cpu().numpy().reshape(T, k), ids)
    assert np.array_equal(b["off"].cpu().numpy(), off)
    assert np.array_equal(b["ps"].cpu().numpy(), ps)
    assert np.array_equal(b["p2r"].cpu().numpy(), p2r)


def test_route_permute_without_tokens(cuda_device):
    b = _buffers(0, 16, 2)
    _lib.route_permute(0, 0, 16, 2, 0, 0, 0, b["off"].data_ptr(), 0, 0, 0, 0, _stream())
    torch.cuda.synchronize()
    assert b["off"].cpu().tolist() == [0] * 17


def test_route_permute_counts_one_launch_on_small_batches(cuda_device):
    T, E, k = 64, 128, 8
    d_lg = torch.from_numpy(_logits(T, E, k, 5, False)).cuda()
    b = _buffers(T, E, k)
    _lib.profile_read(reset=True)
    _lib.route_permute(d_lg.data_ptr(), T, E, k, 0, b["ids"].data_ptr(), b["w"].data_ptr(), b["off"].data_ptr(),
                       b["ps"].data_ptr(), b["p2r"].data_ptr(), 0, 0, _stream())
    torch.cuda.synchronize()
    prof = _lib.profile_read(reset=True)
    assert prof["route_permute"][0] == 1
    assert prof["route"][0] == 0 and prof["permute"][0] == 0


@pytest.mark.parametrize("name", ["tiny", "decode_T64"])
def test_layer_through_the_fused_front(cuda_device, name):
    w = inputs.WORKLOADS[name]
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w)
    run = G.run_gpu(w, pool=pool, slot_table=st, li=li, fused_front=True)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)
