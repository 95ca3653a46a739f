"""CPU oracle, part 2: one MoE FFN layer, written as its plain definition.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module;
only the tests, the package's smoke check and the bench's CPU-baseline leg do.

The pages describe the engine that serves this layer (FlashML-org / FreeToken
About page, "Fast Edge-Native Runtime": MoE serving with a global LRU expert
cache; FreeToken model guide, "MoE expert scheduling strategies") but never
write the layer down.  The plainest reading of a top-k MoE FFN layer with
NVFP4 experts, used here:

  route    S(t) = the k experts with the largest fp32 logits (descending;
           equal logits: lower expert id first);
           w_j  = exp(l_j - m) / sum_{i in S(t)} exp(l_i - m),  m = max_S l
           (softmax over all E followed by renormalising over S, and softmax
           over the k selected logits, are the same function);
  permute  pair p = t*k + j goes to expert ids[p]; groups are contiguous in
           expert order, ordered by ascending p inside a group;
  expert   h = silu(Wg x) * (Wu x),  silu(a) = a / (1 + e^-a);  o = Wd h
           (W* dequantised from NVFP4, x the bf16 activation row);
  combine  y[t] = sum_j w_j * o_{t,j}.

Everything is fp64; no intermediate is rounded to bf16.  Parity pins: see
tests/test_oracle_moe.py (brute-force top-k, permutation invariants, a
one-expert/top-1 case against torch's dense fp64 SwiGLU, closed forms).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional, Sequence

import numpy as np

from . import nvfp4


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> fp64 (exact: bf16 is the top half of an fp32)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


# ----------------------------------------------------------------- route ---

def route(logits: np.ndarray, k: int):
    """Top-k selection on fp32 logits and renormalised fp64 weights.

    Returns ids int32 [T, k] (descending logit, ties -> lower id) and
    w fp64 [T, k].
    """
    lg = np.asarray(logits, dtype=np.float32)
    T, E = lg.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    eid = np.arange(E)
    for t in range(T):
        order = np.lexsort((eid, -lg[t].astype(np.float64)))   # by -logit, then id
        sel = order[:k]
        ids[t] = sel
        l = lg[t, sel].astype(np.float64)
        e = np.exp(l - l.max())
        w[t] = e / e.sum()
    return ids, w


def softmax_then_renorm(logits: np.ndarray, ids: np.ndarray) -> np.ndarray:
    """Weights via softmax over all E and renormalisation over the selected ids."""
    lg = np.asarray(logits, dtype=np.float64)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ps = np.take_along_axis(p, ids.astype(np.int64), axis=1)
    return ps / ps.sum(axis=1, keepdims=True)


# --------------------------------------------------------------- permute ---

def permute(ids: np.ndarray, E: int):
    """Stable counting sort of pairs by expert.

    Returns offsets int32 [E+1], perm_src int32 [T*k] (row -> pair) and
    pair_to_row int32 [T*k] (pair -> row).
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    P = flat.size
    counts = np.zeros(E, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    cursor = offsets[:-1].copy()
    perm_src = np.empty(P, dtype=np.int64)
    for p in range(P):                      # ascending p keeps each group ordered
        e = flat[p]
        perm_src[cursor[e]] = p
        cursor[e] += 1
    pair_to_row = np.empty(P, dtype=np.int64)
    pair_to_row[perm_src] = np.arange(P)
    return offsets.astype(np.int32), perm_src.astype(np.int32), pair_to_row.astype(np.int32)


# ---------------------------------------------------------------- expert ---

@dataclasses.dataclass
class Nvfp4Tensor:
    codes: np.ndarray      # uint8 [N, K/2]
    scales: np.ndarray     # uint8 [N, ld_scale]
    global_scale: float    # fp32
    N: int
    K: int

    def dense(self) -> np.ndarray:
        return nvfp4.decode(self.codes, self.scales, self.global_scale,
                            self.N, self.K, self.scales.shape[1])


@dataclasses.dataclass
class Expert:
    gate: Nvfp4Tensor      # [I, H]
    up: Nvfp4Tensor        # [I, H]
    down: Nvfp4Tensor      # [H, I]


def silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def expert_ffn(x: np.ndarray, ex: Expert) -> np.ndarray:
    """x fp64 [n, H] -> o fp64 [n, H] = Wd (silu(Wg x) * (Wu x))."""
    wg, wu, wd = ex.gate.dense(), ex.up.dense(), ex.down.dense()
    g = x @ wg.T
    u = x @ wu.T
    return (silu(g) * u) @ wd.T


def expert_hidden(x: np.ndarray, ex: Expert) -> np.ndarray:
    """The intermediate h = silu(Wg x) * (Wu x), fp64 [n, I]."""
    return silu(x @ ex.gate.dense().T) * (x @ ex.up.dense().T)


# ----------------------------------------------------------------- layer ---

@dataclasses.dataclass
class LayerResult:
    ids: np.ndarray
    w: np.ndarray
    offsets: np.ndarray
    perm_src: np.ndarray
    pair_to_row: np.ndarray
    out_perm: Optional[np.ndarray]   # fp64 [T*k, H] (None when tokens were sampled)
    y: np.ndarray                    # fp64 [T or len(tokens), H]


def moe_layer(x_bits: np.ndarray, logits: np.ndarray, k: int,
              experts: Dict[int, Expert], tokens: Optional[Sequence[int]] = None,
              keep_out_perm: bool = True) -> LayerResult:
    """The whole layer.  ``experts`` maps expert id -> Expert and needs to hold
    only the experts some evaluated token selects.  With ``tokens`` given, the
    expert FFN and the combine run for those tokens only (route and permute
    always run for every token)."""
    T, E = np.asarray(logits).shape
    x = bf16_bits_to_f64(x_bits)
    ids, w = route(logits, k)
    offsets, perm_src, pair_to_row = permute(ids, E)
    H = x.shape[1]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pairs = (tok[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    o_pair = np.zeros((pairs.size, H), dtype=np.float64)
    pair_expert = ids.reshape(-1)[pairs]
    for e in np.unique(pair_expert):
        sel = np.nonzero(pair_expert == e)[0]
        o_pair[sel] = expert_ffn(x[pairs[sel] // k], experts[int(e)])
    y = (o_pair.reshape(tok.size, k, H) * w[tok][:, :, None]).sum(axis=1)
    out_perm = None
    if tokens is None and keep_out_perm:
        out_perm = np.empty((T * k, H), dtype=np.float64)
        out_perm[pair_to_row[pairs]] = o_pair
    return LayerResult(ids, w, offsets, perm_src, pair_to_row, out_perm, y)


def tolerance(y_ref: np.ndarray) -> float:
    """Per-element bound |y_gpu - y_ref| <= 1e-2 * rms(y_ref) + 1e-3 (rms over
    every element of the layer output)."""
    y = np.asarray(y_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y * y))) if y.size else 0.0
    return 1e-2 * rms + 1e-3
