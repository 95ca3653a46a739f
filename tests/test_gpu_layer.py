"""Whole-layer parity with the oracle through the C ABI, on every workload
family (full outputs where the oracle is quick, sampled tokens at full size),
plus edge cases and exact invariants of the GPU path."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import _lib, inputs
from moe_expert_layer_renorm_b200.layer import MoELayer
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


def _sample(T, n, seed=0):
    if T <= n:
        return None
    g = np.random.default_rng(seed)
    return np.sort(np.concatenate([[0, T - 1], g.choice(np.arange(1, T - 1), size=n - 2, replace=False)]))


@pytest.mark.parametrize("name", ["tiny", "decode_T1", "decode_T8", "decode_T32", "decode_T64"])
def test_layer_full_parity(cuda_device, name):
    w = W[name]
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)


@pytest.mark.parametrize("H,I,E,k,T", [(320, 448, 8, 2, 40), (256, 256, 4, 4, 100), (576, 320, 16, 3, 333),
                                         (320, 448, 4, 2, 600), (576, 2880, 3, 2, 700),
                                         (320, 448, 32, 2, 400), (576, 320, 64, 4, 600)])
def test_ragged_shapes(cuda_device, H, I, E, k, T):
    # K not a multiple of 256, output features not a multiple of 128, groups spanning several tiles; the
    # 4th and 5th have hundreds of rows per expert (the gate/up GEMM's large-group shape), the last two a few
    # dozen (both GEMMs' small-group shape: 64-row token tiles)
    w = inputs.custom_workload(W["tiny"], H=H, I=I, E=E, k=k, T=T, seed=4242 + H)
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    G.check_output(run, w.k)


def test_small_groups_skewed(cuda_device):
    # a few dozen rows per expert on average (the small-group shape) with Zipf-skewed routing, so that some
    # groups take several 64-row tiles and others none
    w = inputs.custom_workload(W["tiny"], H=256, I=512, E=64, k=2, T=700, zipf_s=1.1, seed=4711)
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    counts = np.diff(run.layer.offsets.cpu().numpy())
    assert counts.max() > 128 and counts.min() < 8
    assert 16 < w.T * w.k / max(1, int((counts > 0).sum())) < 48
    G.check_output(run, w.k)


def test_prefill_skewed_sampled(cuda_device):
    w = W["prefill_zipf_T4096"]
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    counts = np.diff(run.layer.offsets.cpu().numpy())
    assert counts.max() > 512 and counts.min() < 64          # skewed: groups span many tiles
    G.check_output(run, w.k, tokens=_sample(w.T, 96, 1))


@pytest.mark.parametrize("name,n", [("slots512_T1", None), ("slots512_T2048", 64)])
def test_slot_pool_indirection(cuda_device, name, n):
    w = W[name]
    run = G.run_gpu(w)
    assert len(set(run.slot_table.tolist())) == w.E and run.slot_table.max() < 4096
    G.check_routing(run, w.k)
    G.check_output(run, w.k, tokens=None if n is None else _sample(w.T, n, 2))


@pytest.mark.slow
def test_slot_pool_T8192_sampled(cuda_device):
    w = W["slots512_T8192"]
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    G.check_output(run, w.k, tokens=_sample(w.T, 48, 3))


def test_wide_experts_sampled(cuda_device):
    w = W["wide_T8192"]
    run = G.run_gpu(w)
    G.check_routing(run, w.k)
    G.check_output(run, w.k, tokens=_sample(w.T, 24, 4))


def test_wide_decode_sweep_layers(cuda_device):
    # every layer of the 48-layer sweep (independent seeded weights and inputs), each checked on its own
    w = W["wide_decode_T1"]
    assert inputs.WIDE_SWEEP_LAYERS == 48
    for layer in range(inputs.WIDE_SWEEP_LAYERS):
        run = G.run_gpu(w, layer=layer)
        G.check_routing(run, w.k)
        G.check_output(run, w.k)
        del run
        torch.cuda.empty_cache()


def test_all_tokens_one_expert(cuda_device):
    # one group of 3 * 128 + 5 rows: several token tiles and a ragged tail
    w = inputs.custom_workload(W["tiny"], T=389, seed=77)
    li = inputs.make_layer_inputs(w)
    li.logits[:, 3] += 50.0
    run = G.run_gpu(w, li=li)
    G.check_routing(run, w.k)
    assert np.diff(run.layer.offsets.cpu().numpy())[3] == w.T
    G.check_output(run, w.k)


def test_top1_single_expert(cuda_device):
    w = inputs.custom_workload(W["tiny"], E=1, k=1, T=50, seed=91)
    run = G.run_gpu(w)
    G.check_routing(run, 1)
    G.check_output(run, 1)


def test_zero_tokens_is_a_noop(cuda_device):
    lay = MoELayer(0, 8, 2, 256, 512)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    lg = torch.empty((0, 8), dtype=torch.float32, device="cuda")
    pool, st = G.build_pool(W["tiny"])
    y = lay.forward(x, lg, torch.from_numpy(st).cuda(), pool)
    torch.cuda.synchronize()
    assert y.shape == (0, 256)
    assert lay.offsets.cpu().numpy().tolist() == [0] * 9


def test_reruns_are_bit_identical(cuda_device):
    w = W["decode_T64"]
    run = G.run_gpu(w)
    first = run.layer.y.clone()
    x = torch.from_numpy(run.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    lg = torch.from_numpy(run.logits).cuda()
    st = torch.from_numpy(run.slot_table.astype(np.int32)).cuda()
    for _ in range(3):
        y = run.layer.forward(x, lg, st, run.pool)
        torch.cuda.synchronize()
        assert torch.equal(y, first)


def test_relabelled_slot_table_is_bit_identical(cuda_device):
    w = W["tiny"]
    run = G.run_gpu(w)
    # move every expert to another slot of a larger pool
    w2 = inputs.custom_workload(w, n_slots=64)
    pool2 = G.ExpertPool(w.H, w.I, 64)
    g = np.random.default_rng(5)
    st2 = g.permutation(64)[: w.E].astype(np.int32)
    for e in range(w.E):
        pool2.slot_view(int(st2[e])).copy_(run.pool.slot_view(int(run.slot_table[e])))
    run2 = G.run_gpu(w2, pool=pool2, slot_table=st2)
    assert np.array_equal(run.y, run2.y)


def test_down_global_scale_doubles_output_exactly(cuda_device):
    w = W["decode_T8"]
    run = G.run_gpu(w)
    L = run.pool.layout
    for slot in range(run.pool.num_slots):
        off = slot * run.pool.slot_bytes + L.global_off[_lib.FT_DOWN]
        view = run.pool.buf[off:off + 4].view(torch.float32)
        view.mul_(2.0)
    run2 = G.run_gpu(w, pool=run.pool, slot_table=run.slot_table)
    assert np.array_equal(run2.y, 2.0 * run.y)


def test_non_resident_expert_sets_status(cuda_device):
    w = W["tiny"]
    _lib.device_status(clear=True)
    li = inputs.make_layer_inputs(w)
    pool, st = G.build_pool(w)
    ids, _ = G.M.route(li.logits, w.k)
    st = st.copy()
    st[int(ids[0, 0])] = -1
    G.run_gpu(w, pool=pool, slot_table=st, li=li, expect_status=_lib.FT_DEV_NOT_RESIDENT)
    # the library stays usable afterwards
    run = G.run_gpu(w)
    G.check_output(run, w.k)
    assert _lib.device_status(clear=True) == _lib.FT_DEV_OK


def test_cuda_graph_capture_replays_the_layer(cuda_device):
    w = W["decode_T32"]
    run = G.run_gpu(w)
    ref = run.layer.y.clone()
    x = torch.from_numpy(run.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    lg = torch.from_numpy(run.logits).cuda()
    st = torch.from_numpy(run.slot_table.astype(np.int32)).cuda()
    s = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        run.layer.forward(x, lg, st, run.pool, stream=s)   # warm the launch path outside capture
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            run.layer.forward(x, lg, st, run.pool, stream=s)
    run.layer.y.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(run.layer.y, ref)
