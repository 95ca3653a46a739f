"""Expert-cache churn on the GPU: layers whose experts are brought into a small
device pool by the slot manager (misses, evictions across layers, fills that
overlap the previous layer's kernels) give bit-identical outputs to the same
layers run with every expert resident."""
import numpy as np
import pytest
import torch

from moe_expert_layer_renorm_b200 import churn
from moe_expert_layer_renorm_b200.layer import MoELayer


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["demand", "prefetch"])
def test_churn_matches_resident(cuda_device, mode):
    # 4 layers x up to 6 distinct experts per call, 18 slots: most steps
    # evict slots of other layers, some of them read by the previous layer
    # (a host run of the same policy: 16 hits, 104 misses, 86 evictions)
    cfg = churn.ChurnConfig(T=4, E=16, k=2, H=256, I=512, layers=4, domains=2, hot=6, capacity=18)
    hs = churn.hot_sets(cfg)
    banks = churn.ExpertBanks(cfg, hs, keep_device=True)
    run = churn.ChurnRun(cfg, banks)
    outs, all_logits = [], []
    for step, d in enumerate([0, 0, 1, 1, 0, 1]):
        logits = [torch.from_numpy(churn.step_logits(cfg, hs, l, d, step)).cuda() for l in range(cfg.layers)]
        all_logits.append(logits)
        run.step(logits, mode, outs)
    torch.cuda.synchronize()
    st = run.mgr.stats()
    assert st["misses"] > 0 and st["evictions"] > 0 and st["hits"] > 0
    ref = MoELayer(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I)
    i = 0
    for logits in all_logits:
        for l in range(cfg.layers):
            y = ref.forward(run.x[l], logits[l], banks.resident_table(cfg, l), banks.resident)
            torch.cuda.synchronize()
            assert torch.equal(y, outs[i]), f"layer {l}, output {i}"
            assert torch.isfinite(y).all()
            i += 1
    run.mgr.close()


def test_churn_routes_to_hot_sets():
    """The domain bias sends every selection into the current domain's hot set
    (host-side inputs only)."""
    cfg = churn.ChurnConfig(T=8, E=32, k=4, H=256, I=512, layers=2, domains=3, hot=8, capacity=16)
    hs = churn.hot_sets(cfg)
    assert len(set(hs[0].ravel().tolist())) == cfg.domains * cfg.hot   # disjoint hot sets
    for d in range(cfg.domains):
        lg = churn.step_logits(cfg, hs, 1, d, 5)
        top = np.argsort(-lg, axis=1)[:, :cfg.k]
        assert set(top.ravel().tolist()) <= set(hs[1, d].tolist())


@pytest.mark.gpu
def test_prefill_streaming_matches_resident(cuda_device):
    # the prefill streaming order: 3 layers of 512 tokens, every expert of a
    # layer used (k = 4 of E = 16, one domain), a pool of two layers' worth,
    # so each layer's 16 experts are filled from the host while the previous
    # layer runs, evicting the slots of the layer before it; the groups (~128
    # rows per expert) take the tcgen05 kernels.  Outputs are bit-identical to
    # the same layers with every expert resident, and the fills coalesce.
    cfg = churn.ChurnConfig(T=512, E=16, k=4, H=256, I=256, layers=3, domains=1, hot=16, capacity=32)
    hs = churn.hot_sets(cfg)
    banks = churn.ExpertBanks(cfg, hs, keep_device=True)
    run = churn.ChurnRun(cfg, banks)
    outs, all_logits = [], []
    for step in range(3):
        logits = [torch.from_numpy(churn.step_logits(cfg, hs, l, 0, step)).cuda() for l in range(cfg.layers)]
        all_logits.append(logits)
        run.step(logits, "prefetch", outs)
    torch.cuda.synchronize()
    st = run.mgr.stats()
    assert st["misses"] == 16 * 3 * 3 and st["evictions"] > 0
    assert st["copies"] < st["misses"]          # runs of consecutive slots and banks
    ref = MoELayer(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I)
    i = 0
    for logits in all_logits:
        for l in range(cfg.layers):
            y = ref.forward(run.x[l], logits[l], banks.resident_table(cfg, l), banks.resident)
            torch.cuda.synchronize()
            assert torch.equal(y, outs[i]), f"layer {l}, output {i}"
            assert torch.isfinite(y).all()
            i += 1
    run.mgr.close()
