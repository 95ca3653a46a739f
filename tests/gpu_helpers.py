"""Shared set-up for the GPU parity tests: build an expert pool from the
seeded generators, run the layer through the C ABI, and build the oracle's
view of the same experts from the packed bytes downloaded from the pool."""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np
import torch

from moe_expert_layer_renorm_b200 import inputs
from moe_expert_layer_renorm_b200.layer import ExpertPool, MoELayer
from oracle import moe_layer as M


def build_pool(w: inputs.Workload, layer: int = 0, device="cuda", fmt: int = 0, tiled: bool = False):
    s = inputs.layer_seed(w.seed, layer)
    slot_table = inputs.make_slot_table(w.E, w.slots, w.permuted_slots, s)
    pool = ExpertPool(w.H, w.I, w.slots, device=device, fmt=fmt, tiled=tiled)
    for e in range(w.E):
        for mat in range(3):
            N, K = pool.shape(mat)
            wt = inputs.make_weight_fp32_torch(N, K, s, e, mat, device)
            pool.pack_into(int(slot_table[e]), mat, wt)
    torch.cuda.synchronize()
    return pool, slot_table


def oracle_experts(pool: ExpertPool, slot_table: np.ndarray, experts) -> dict:
    out = {}
    for e in sorted(set(int(v) for v in experts)):
        mats = []
        for mat in range(3):
            c, sc, g = pool.tensor_bytes(int(slot_table[e]), mat)
            N, K = pool.shape(mat)
            mats.append(M.Nvfp4Tensor(c, sc, g, N, K))
        out[e] = M.Expert(*mats)
    return out


@dataclasses.dataclass
class GpuRun:
    layer: MoELayer
    x_bits: np.ndarray
    logits: np.ndarray
    slot_table: np.ndarray
    pool: ExpertPool
    y: np.ndarray          # fp64 copy of the bf16 output


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def _a256(n: int) -> int:
    return (n + 255) // 256 * 256


def poison(lay: MoELayer) -> None:
    """Fill what the layer writes before it reads with NaN (0xFF bytes): the
    outputs, the separate calls' FFN workspace, and the data part of the
    whole-layer workspace (its f16 token rows, row factors and h, which come
    before its counters; the counters must stay zero)."""
    lay.out_perm.fill_(float("nan"))
    lay.y.fill_(float("nan"))
    if lay.whole:
        T, k, H, I = lay.T, lay.k, lay.H, lay.I
        data = _a256(T * H * 2) + _a256(T * 4) + _a256(T * k * I * 2)
        ws = lay.layer_ws
        ws[:min(data, ws.numel())].fill_(0xFF)
    else:
        lay.ffn_ws.fill_(0xFF)


def run_gpu(w: inputs.Workload, T: Optional[int] = None, layer: int = 0, pool=None, slot_table=None,
            li: Optional[inputs.LayerInputs] = None, expect_status: int = 0, fused_front: bool = False,
            whole: bool = False) -> GpuRun:
    li = li or inputs.make_layer_inputs(w, layer, T)
    T = li.x_bits.shape[0]
    if pool is None:
        pool, slot_table = build_pool(w, layer)
    x = torch.from_numpy(li.x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    logits = torch.from_numpy(li.logits).cuda()
    st = torch.from_numpy(np.asarray(slot_table, dtype=np.int32)).cuda()
    lay = MoELayer(T, w.E, w.k, w.H, w.I, mode=w.route_mode, fused_front=fused_front, whole=whole)
    # NaN in every intermediate the library writes before reading: an element
    # read before it is written (a missed dependency) shows up in y
    poison(lay)
    from moe_expert_layer_renorm_b200 import _lib
    _lib.device_status(clear=True)
    y = lay.forward(x, logits, st, pool)
    torch.cuda.synchronize()
    detail = _lib.device_status_detail()
    status = _lib.device_status(clear=True)
    assert status == expect_status, f"device status {status} (detail {detail})"
    return GpuRun(lay, li.x_bits, li.logits, np.asarray(slot_table), pool, bf16_to_f64(y))


def check_routing(run: GpuRun, k: int):
    """ids, offsets, perm_src, pair_to_row bit-exact; weights to fp32 rounding."""
    ids, w = M.route(run.logits, k)
    E = run.logits.shape[1]
    off, ps, p2r = M.permute(ids, E)
    L = run.layer
    assert np.array_equal(L.ids.cpu().numpy(), ids)
    assert np.allclose(L.w.cpu().numpy().astype(np.float64), w, rtol=2e-6, atol=1e-7)
    assert np.array_equal(L.offsets.cpu().numpy(), off)
    assert np.array_equal(L.perm_src.cpu().numpy(), ps)
    assert np.array_equal(L.pair_to_row.cpu().numpy(), p2r)
    return ids


def host_pool(pool: ExpertPool, slot_table: np.ndarray, experts):
    """The slots of the given experts copied to the host, packed densely, and
    the slot table that points into that copy (-1 for the other experts)."""
    need = sorted(set(int(v) for v in experts))
    L = pool.rows_layout           # slots read back in the row-major layout
    nb = int(L.slot_bytes)
    buf = np.zeros(max(1, len(need)) * nb, np.uint8)
    table = np.full(len(slot_table), -1, np.int32)
    for i, e in enumerate(need):
        buf[i * nb:(i + 1) * nb] = pool.export_slot(int(slot_table[e]))
        table[e] = i
    return buf, table, L


def reference_y(run: GpuRun, k: int, tok: np.ndarray) -> np.ndarray:
    """The C++ oracle's y for the tokens `tok`, from the packed bytes in the pool."""
    from oracle import cpp
    ids = run.layer.ids.cpu().numpy()
    buf, table, L = host_pool(run.pool, run.slot_table, ids[tok].reshape(-1))
    H, I = run.pool.H, run.pool.I
    return cpp.moe_layer(run.x_bits, run.logits, k, table, buf, int(L.slot_bytes), list(L.codes_off),
                         list(L.scales_off), list(L.global_off), list(L.ld_scale), H, I, tokens=tok,
                         fmt=int(L.scale_format))


def check_output(run: GpuRun, k: int, tokens: Optional[Sequence[int]] = None):
    """y within 1e-2 * rms(y_ref) + 1e-3 element-wise (rms over the evaluated tokens)."""
    T = run.x_bits.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens)
    ref_y = reference_y(run, k, tok)
    y = run.y[tok]
    tol = M.tolerance(ref_y)
    err = np.abs(y - ref_y)
    worst = float(err.max()) if err.size else 0.0
    assert np.all(err <= tol), f"max |err| {worst:.3g} > tol {tol:.3g} (rms {np.sqrt(np.mean(ref_y ** 2)):.3g})"
    return worst, tol
