"""Seeded synthetic inputs for the NVFP4 MoE FFN layer.

This module only draws random numbers and arranges them into the shapes the
layer consumes; it performs none of the layer's arithmetic (no routing, no
quantisation, no GEMM).  Both the CUDA path's tests/bench and the CPU oracle's
tests take their inputs from here, so the two sides always see identical bytes.

The pages describe a serving engine for NVFP4 MoE models (FreeToken model
guide, "MoE expert scheduling strategies"; sm89-moe-offload fork README,
"Production configuration") but publish no dataset for the layer itself, so
every workload is synthetic:

* activations x: bf16, round-to-nearest-even of N(0, 1) fp32 draws;
* router logits: fp32 N(0, sigma) (+ an optional per-expert bias), re-drawn
  per token until the gap between the k-th and (k+1)-th largest logit exceeds
  ``min_gap`` so that the selected set is unambiguous in fp32;
* expert weights: fp32 N(0, 0.02), generated per expert with a seeded torch
  generator (on the device for large workloads), then packed to NVFP4.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

ROUTE_SOFTMAX_RENORM = 0  # softmax over all E logits, keep top-k, renormalise
ROUTE_TOPK_SOFTMAX = 1    # keep top-k logits, softmax over the k of them

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic MoE layer configuration."""
    name: str
    T: int
    E: int
    k: int
    H: int
    I: int
    route_mode: int = ROUTE_SOFTMAX_RENORM
    logit_sigma: float = 1.0
    zipf_s: Optional[float] = None      # per-expert Zipf-ranked logit bias
    zipf_span: float = 2.0              # bias mapped onto [-span, +span]
    n_slots: Optional[int] = None       # slot pool size (None: one slot per expert)
    permuted_slots: bool = False        # random injective expert -> slot map
    seed: int = 1000

    @property
    def slots(self) -> int:
        return self.n_slots if self.n_slots is not None else self.E


def _base(idx: int) -> int:
    return 1000 + idx


# The five layer families (tiny parity layer, decode, Zipf-skewed prefill,
# large expert count behind a 4096-slot pool, wide experts).
WORKLOADS = {
    "tiny": Workload("tiny", T=16, E=8, k=2, H=256, I=512, seed=_base(0)),
    **{f"decode_T{t}": Workload(f"decode_T{t}", T=t, E=128, k=8, H=2048, I=768, seed=_base(1))
       for t in (1, 8, 32, 64)},
    "prefill_zipf_T4096": Workload("prefill_zipf_T4096", T=4096, E=128, k=8, H=2048, I=768,
                                   zipf_s=1.1, seed=_base(2)),
    **{f"slots512_T{t}": Workload(f"slots512_T{t}", T=t, E=512, k=10, H=2048, I=512,
                                  n_slots=4096, permuted_slots=True, seed=_base(3))
       for t in (1, 2048, 8192)},
    "wide_T8192": Workload("wide_T8192", T=8192, E=32, k=4, H=2880, I=2880,
                           route_mode=ROUTE_TOPK_SOFTMAX, logit_sigma=1.5, seed=_base(4)),
    "wide_decode_T1": Workload("wide_decode_T1", T=1, E=32, k=4, H=2880, I=2880,
                               route_mode=ROUTE_TOPK_SOFTMAX, logit_sigma=1.5, seed=_base(4)),
}

WIDE_SWEEP_LAYERS = 48


def layer_seed(seed: int, layer: int) -> int:
    """Seed of layer ``layer`` in a multi-layer sweep."""
    return seed + 7919 * layer


def rng(seed: int, stream: int) -> np.random.Generator:
    """Independent numpy PCG64 stream ``stream`` of ``seed``."""
    return np.random.Generator(np.random.PCG64([seed, stream]))


def fp32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_fp32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_x_bits(T: int, H: int, seed: int) -> np.ndarray:
    """Activations as bf16 bit patterns, uint16 [T, H]."""
    g = rng(seed, 1)
    return fp32_to_bf16_bits(g.standard_normal((T, H), dtype=np.float32))


def zipf_bias(E: int, s: float, span: float, seed: int) -> np.ndarray:
    """Per-expert logit bias from a Zipf(s) ranking.

    A random permutation gives each expert a rank r in 1..E; z = r**-s and
    log z is mapped affinely onto [-span, +span] (rank 1 -> +span).
    """
    g = rng(seed, 3)
    rank = g.permutation(E) + 1
    lz = -s * np.log(rank.astype(np.float64))
    lo, hi = -s * math.log(E), 0.0
    b = -span + (lz - lo) * (2.0 * span / (hi - lo))
    return b.astype(np.float32)


def make_logits(T: int, E: int, k: int, sigma: float, seed: int,
                bias: Optional[np.ndarray] = None, min_gap: float = 1e-4) -> np.ndarray:
    """Router logits fp32 [T, E] with an unambiguous top-k boundary per token."""
    g = rng(seed, 2)
    out = np.empty((T, E), dtype=np.float32)
    b = np.zeros(E, np.float32) if bias is None else bias.astype(np.float32)
    todo = np.arange(T)
    while todo.size:
        draw = (g.standard_normal((todo.size, E), dtype=np.float32) * np.float32(sigma)) + b
        out[todo] = draw
        if k >= E:
            break
        srt = -np.sort(-draw, axis=1)
        ok = (srt[:, k - 1] - srt[:, k]) > np.float32(min_gap)
        todo = todo[~ok]
    return out


def make_slot_table(E: int, n_slots: int, permuted: bool, seed: int) -> np.ndarray:
    """expert -> slot map, int32 [E]; identity or a seeded injective map."""
    if not permuted:
        assert n_slots >= E
        return np.arange(E, dtype=np.int32)
    g = rng(seed, 4)
    return g.permutation(n_slots)[:E].astype(np.int32)


def make_weight_fp32_host(rows: int, cols: int, seed: int, expert: int, which: int) -> np.ndarray:
    """fp32 N(0, 0.02) weights drawn on the host (small workloads and CPU tests)."""
    g = np.random.Generator(np.random.PCG64([seed, 100 + which, expert]))
    return (g.standard_normal((rows, cols), dtype=np.float32) * np.float32(WEIGHT_STD))


def make_weight_fp32_torch(rows: int, cols: int, seed: int, expert: int, which: int, device):
    """fp32 N(0, 0.02) weights drawn by a seeded torch generator on ``device``."""
    import torch
    gen = torch.Generator(device=device)
    gen.manual_seed((seed * 1_000_003 + expert * 31 + which) & 0x7FFF_FFFF_FFFF)
    w = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32)
    return w.mul_(WEIGHT_STD)


@dataclasses.dataclass
class LayerInputs:
    x_bits: np.ndarray      # uint16 [T, H] bf16 bit patterns
    logits: np.ndarray      # fp32 [T, E]
    slot_table: np.ndarray  # int32 [E]


def make_layer_inputs(w: Workload, layer: int = 0, T: Optional[int] = None) -> LayerInputs:
    s = layer_seed(w.seed, layer)
    T = w.T if T is None else T
    bias = zipf_bias(w.E, w.zipf_s, w.zipf_span, s) if w.zipf_s else None
    return LayerInputs(
        x_bits=make_x_bits(T, w.H, s),
        logits=make_logits(T, w.E, w.k, w.logit_sigma, s, bias=bias),
        slot_table=make_slot_table(w.E, w.slots, w.permuted_slots, s),
    )


def expected_distinct_experts(T: int, E: int, k: int) -> float:
    """Expected number of distinct experts hit by T uniformly routed tokens."""
    return E * (1.0 - (1.0 - k / E) ** T)


def custom_workload(base: Workload, **kw) -> Workload:
    return dataclasses.replace(base, **kw)


__all__: Sequence[str] = [
    "Workload", "WORKLOADS", "ROUTE_SOFTMAX_RENORM", "ROUTE_TOPK_SOFTMAX", "WIDE_SWEEP_LAYERS",
    "make_layer_inputs", "make_x_bits", "make_logits", "make_slot_table", "zipf_bias",
    "make_weight_fp32_host", "make_weight_fp32_torch", "fp32_to_bf16_bits", "bf16_bits_to_fp32",
    "layer_seed", "expected_distinct_experts", "custom_workload",
]
