"""Expert-cache churn: a multi-layer decode loop whose experts live in pinned
host banks and are brought into a smaller device pool on demand by the slot
manager (ft_slot_*), under a domain-rotation routing pattern.

The cache mirrors the engine's global LRU expert cache keyed by (layer,
expert) (FreeToken model guide, offload strategy; sm89-moe-offload README,
--moe-cache-size): a miss is one host-to-device copy of the expert's slot
image on a copy stream, and the layer's kernels wait for it.

Workload.  Every layer has E experts.  Domain d owns a hot set of `hot`
experts per layer (disjoint across domains, a seeded permutation per layer).
All tokens of a step belong to the current domain: their logits are N(0, 1)
plus `boost` on that domain's hot set, so a step routes (almost) only to hot
experts, steady steps of a domain hit the cache, and the first step after a
domain switch misses on the new domain's experts.

Two orders of work per step:
  demand    route layer l, read its expert ids on the host, acquire, run the
            layer: a miss is paid in full before the layer starts;
  prefetch  route every layer of the step first (the ids of all layers are
            known at the start of the step, as with a perfect predictor), then
            acquire layer l + 1 while layer l runs, so its fills overlap
            layer l's kernels (the slot manager orders a fill only after the
            last kernels that read the slot it reuses).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np
import torch

from . import inputs
from .layer import ExpertPool, MoELayer, SlotManager


@dataclasses.dataclass
class ChurnConfig:
    T: int
    E: int
    k: int
    H: int
    I: int
    layers: int
    domains: int
    hot: int                 # hot experts per layer per domain
    capacity: int            # device pool slots shared by all layers
    boost: float = 6.0
    seed: int = 4242

    def __post_init__(self):
        assert self.domains * self.hot <= self.E and self.hot >= self.k


def hot_sets(cfg: ChurnConfig) -> np.ndarray:
    """int32 [layers, domains, hot]: the experts each domain favours per layer."""
    out = np.empty((cfg.layers, cfg.domains, cfg.hot), np.int32)
    for l in range(cfg.layers):
        perm = inputs.rng(inputs.layer_seed(cfg.seed, l), 7).permutation(cfg.E)
        out[l] = perm[:cfg.domains * cfg.hot].reshape(cfg.domains, cfg.hot)
    return out


def step_logits(cfg: ChurnConfig, hs: np.ndarray, layer: int, domain: int, step: int) -> np.ndarray:
    """Router logits fp32 [T, E] of one layer in one step of `domain`."""
    bias = np.zeros(cfg.E, np.float32)
    bias[hs[layer, domain]] = np.float32(cfg.boost)
    return inputs.make_logits(cfg.T, cfg.E, cfg.k, 1.0, inputs.layer_seed(cfg.seed + 17 * step, layer), bias=bias)


class ExpertBanks:
    """Page-locked host images (slot_bytes each) of every (layer, expert) that
    a hot set contains, packed on the device once and copied down.  With
    keep_device the packed device pool stays (bank b in slot b), as the fully
    resident reference."""

    def __init__(self, cfg: ChurnConfig, hs: np.ndarray, keep_device: bool = False, device="cuda"):
        self.keys: List[tuple] = []
        for l in range(cfg.layers):
            for e in sorted(set(int(v) for v in hs[l].ravel())):
                self.keys.append((l, e))
        self.index: Dict[tuple, int] = {key: i for i, key in enumerate(self.keys)}
        n = len(self.keys)
        pool = ExpertPool(cfg.H, cfg.I, n, device=device)
        for i, (l, e) in enumerate(self.keys):
            s = inputs.layer_seed(cfg.seed, l)
            for mat in range(3):
                N, K = pool.shape(mat)
                pool.pack_into(i, mat, inputs.make_weight_fp32_torch(N, K, s, e, mat, device))
        torch.cuda.synchronize()
        self.slot_bytes = pool.slot_bytes
        self.host = torch.empty((n, self.slot_bytes), dtype=torch.uint8).pin_memory()
        self.host.copy_(pool.buf.view(n, self.slot_bytes))
        self.resident: Optional[ExpertPool] = pool if keep_device else None
        if not keep_device:
            del pool
            torch.cuda.empty_cache()

    def ptr(self, layer: int, expert: int) -> int:
        return self.host[self.index[(layer, expert)]].data_ptr()

    def resident_table(self, cfg: ChurnConfig, layer: int) -> torch.Tensor:
        """slot table [E] of `layer` into the resident pool (-1 off the hot sets)."""
        t = np.full(cfg.E, -1, np.int32)
        for (l, e), i in self.index.items():
            if l == layer:
                t[e] = i
        return torch.from_numpy(t).cuda()


class ChurnRun:
    """The device pool, the slot manager and one MoELayer (buffers) per layer."""

    def __init__(self, cfg: ChurnConfig, banks: ExpertBanks, device="cuda"):
        self.cfg = cfg
        self.pool = ExpertPool(cfg.H, cfg.I, cfg.capacity, device=device)
        self.mgr = SlotManager(cfg.capacity, self.pool.layout, self.pool.ptr)
        for (l, e) in banks.keys:
            self.mgr.register_host(l, e, banks.ptr(l, e))
        self.layers = [MoELayer(cfg.T, cfg.E, cfg.k, cfg.H, cfg.I) for _ in range(cfg.layers)]
        self.tables = [torch.full((cfg.E,), -1, dtype=torch.int32, device=device) for _ in range(cfg.layers)]
        g = torch.Generator().manual_seed(cfg.seed)
        self.x = [torch.randn((cfg.T, cfg.H), generator=g).to(torch.bfloat16).to(device) for _ in range(cfg.layers)]
        self.compute = torch.cuda.current_stream()
        self.copy = torch.cuda.Stream()

    def _acquire(self, l: int, ids: np.ndarray) -> None:
        self.mgr.acquire(l, ids.ravel().tolist(), self.tables[l].data_ptr(), self.cfg.E,
                         self.compute.cuda_stream, self.copy.cuda_stream)

    def _run_layer(self, l: int) -> None:
        lay = self.layers[l]
        lay.permute(self.compute)
        lay.ffn(self.x[l], self.tables[l], self.pool, self.compute)
        lay.combine(self.compute)

    def step(self, logits: List[torch.Tensor], mode: str, outputs: Optional[list] = None) -> None:
        """One decode step through every layer.  logits[l]: device fp32 [T, E]."""
        L = self.cfg.layers
        if mode == "prefetch":
            for l in range(L):
                self.layers[l].route(logits[l], self.compute)
            ids = [lay.ids.cpu().numpy() for lay in self.layers]   # one host sync for the step
            self._acquire(0, ids[0])
            for l in range(L):
                self._run_layer(l)
                if outputs is not None:
                    outputs.append(self.layers[l].y.clone())
                if l + 1 < L:
                    self._acquire(l + 1, ids[l + 1])   # fills overlap layer l's kernels
        elif mode == "demand":
            for l in range(L):
                self.layers[l].route(logits[l], self.compute)
                self._acquire(l, self.layers[l].ids.cpu().numpy())
                self._run_layer(l)
                if outputs is not None:
                    outputs.append(self.layers[l].y.clone())
        else:
            raise ValueError(mode)


def run_churn(cfg: ChurnConfig, mode: str, steps_per_domain: int, rounds: int, banks: ExpertBanks,
              device="cuda") -> dict:
    """Time `rounds` passes over all domains, `steps_per_domain` steps each.
    Returns per-step device times split into switch steps (the first of a
    domain) and steady steps, and the slot statistics."""
    hs = hot_sets(cfg)
    run = ChurnRun(cfg, banks, device)
    # warm-up: one pass over the domains (fills the pool, builds the kernels' plans)
    order = [d for _ in range(rounds + 1) for d in range(cfg.domains)]
    switch_ms, steady_ms, miss_counts, h2d = [], [], [], []
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step_idx = 0
    for n, d in enumerate(order):
        for s in range(steps_per_domain):
            logits = [torch.from_numpy(step_logits(cfg, hs, l, d, step_idx)).to(device)
                      for l in range(cfg.layers)]
            torch.cuda.synchronize()
            before = run.mgr.stats()
            ev0.record(run.compute)
            run.step(logits, mode)
            ev1.record(run.compute)
            torch.cuda.synchronize()
            after = run.mgr.stats()
            step_idx += 1
            if n < cfg.domains:
                continue   # warm-up pass
            ms = ev0.elapsed_time(ev1)
            (switch_ms if s == 0 else steady_ms).append(ms)
            if s == 0:
                miss_counts.append(after["misses"] - before["misses"])
                h2d.append(after["bytes_h2d"] - before["bytes_h2d"])
    st = run.mgr.stats()
    run.mgr.close()
    return {"switch_ms": switch_ms, "steady_ms": steady_ms, "misses_per_switch": miss_counts,
            "h2d_bytes_per_switch": h2d, "stats": st}


def run_stream(cfg: ChurnConfig, steps: int, banks: ExpertBanks, device="cuda") -> dict:
    """Streaming: every layer of every step needs experts that are not on the
    device (a pool of two layers' worth shared by `layers` > 2 layers), so
    each layer's experts are filled while the previous layer runs (prefetch
    order, a double-buffered pool).  Also times the same steps with every
    expert resident (banks.resident) and the fills alone."""
    assert banks.resident is not None
    hs = hot_sets(cfg)
    run = ChurnRun(cfg, banks, device)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream_ms, resident_ms, h2d = [], [], []
    tables = [banks.resident_table(cfg, l) for l in range(cfg.layers)]
    for step in range(steps + 1):
        logits = [torch.from_numpy(step_logits(cfg, hs, l, 0, step)).to(device) for l in range(cfg.layers)]
        torch.cuda.synchronize()
        before = run.mgr.stats()
        ev0.record(run.compute)
        run.step(logits, "prefetch")
        ev1.record(run.compute)
        torch.cuda.synchronize()
        after = run.mgr.stats()
        if step > 0:
            stream_ms.append(ev0.elapsed_time(ev1))
            h2d.append(after["bytes_h2d"] - before["bytes_h2d"])
        ev0.record(run.compute)
        for l in range(cfg.layers):
            run.layers[l].forward(run.x[l], logits[l], tables[l], banks.resident, run.compute)
        ev1.record(run.compute)
        torch.cuda.synchronize()
        if step > 0:
            resident_ms.append(ev0.elapsed_time(ev1))
    # the fills alone: the same bytes as one step, slot images from the banks
    n = min(cfg.capacity, banks.host.shape[0])
    with torch.cuda.stream(run.copy):
        ev0.record(run.copy)
        for i in range(n):
            run.pool.slot_view(i).copy_(banks.host[i], non_blocking=True)
        ev1.record(run.copy)
    torch.cuda.synchronize()
    copy_gbps = n * banks.slot_bytes / (ev0.elapsed_time(ev1) * 1e6)
    st = run.mgr.stats()
    run.mgr.close()
    return {"stream_ms": stream_ms, "resident_ms": resident_ms, "h2d_bytes_per_step": h2d,
            "copy_only_GBps": copy_gbps, "stats": st}


__all__ = ["ChurnConfig", "ExpertBanks", "ChurnRun", "hot_sets", "step_logits", "run_churn", "run_stream"]
