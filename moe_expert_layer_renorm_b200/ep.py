"""Expert parallelism: one MoE layer whose experts are split over the ranks of
a process group, the rows of each rank's experts exchanged all-to-all.

The fork's production configuration runs every MoE layer with its experts
split over two GPUs ("sm89-moe-offload" fork README, "Production
configuration": --moe-ep-size 2 beside tensor parallelism).  The pages do not
say how the rows travel; the reading used here (ownership in contiguous
blocks, all-to-all of the routed rows, rows back to their owner for the
combine) is spelled out with ft_ep_plan in include/ftmoe.h.

One step on every rank, for its own T tokens:

  1. route and permute over all E experts (ft_moe_route, ft_moe_permute);
  2. lay out one activation row per routed pair in permuted order
     (ft_gather_rows, idx = perm_src, div = k): the rows for rank d are then
     the contiguous range of d's experts;
  3. all-gather the G expert_offsets arrays and build the exchange plan on
     the host (ft_ep_plan); this is the one host synchronisation of the step,
     as the all-to-all needs its split sizes on the host;
  4. all-to-all the activation rows;
  5. ft_moe_ffn_nvfp4 over the local experts on the received rows, read in
     place through the plan's perm_src (k = 1, E = E / G);
  6. put the outputs back in arrival order (ft_gather_rows, idx = ret_idx)
     and all-to-all them back: each rank's out_perm then holds, row for row,
     what one GPU computes for its tokens;
  7. combine (ft_moe_combine).

Every step that touches the layer's data runs in libftmoe.so; this module
moves pointers, sizes and the collective calls (torch.distributed over NCCL
on GPUs).  The collectives carry plain device buffers; no kernel here reads
another GPU's memory.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

from . import _lib
from .layer import ExpertPool, MoELayer, _stream


def owned_experts(E: int, G: int, rank: int) -> range:
    """The experts rank `rank` of G owns: a contiguous block of E / G."""
    if E % G:
        raise ValueError(f"E = {E} is not a multiple of the {G} ranks")
    n = E // G
    return range(rank * n, (rank + 1) * n)


class ExchangePlan:
    """ft_ep_plan's result for one step: host split sizes and the receiver's
    index arrays (host int32 numpy)."""

    def __init__(self, all_offsets: np.ndarray, G: int, E: int, rank: int):
        all_offsets = np.ascontiguousarray(all_offsets, dtype=np.int32)
        assert all_offsets.shape == (G, E + 1)
        self.G, self.E, self.rank = G, E, rank
        self.send_rows = np.zeros(G, np.int32)
        self.recv_rows = np.zeros(G, np.int32)
        self.local_offsets = np.zeros(E // G + 1, np.int32)
        n = _lib.ep_plan(all_offsets, G, E, rank, 0, self.send_rows, self.recv_rows, self.local_offsets, None,
                         None)
        self.n_recv = n
        self.perm_src_local = np.zeros(max(n, 1), np.int32)
        self.ret_idx = np.zeros(max(n, 1), np.int32)
        _lib.ep_plan(all_offsets, G, E, rank, n, self.send_rows, self.recv_rows, self.local_offsets,
                     self.perm_src_local, self.ret_idx)


class DistExchange:
    """The exchange's transport over torch.distributed (NCCL between GPUs,
    gloo between host processes).  Every rank makes the same calls in the
    same order."""

    def __init__(self, group=None):
        self.group = group
        self.world_size = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def gather_offsets(self, offsets: torch.Tensor) -> np.ndarray:
        """All-gather every rank's expert_offsets [E+1]; returns host int32
        [G, E+1] (waits for the gather: the all-to-alls' split sizes come
        from it)."""
        parts = [torch.empty_like(offsets) for _ in range(self.world_size)]
        dist.all_gather(parts, offsets.contiguous(), group=self.group)
        return torch.stack(parts).cpu().numpy().astype(np.int32)

    def rows(self, out: torch.Tensor, inp: torch.Tensor, out_rows, in_rows) -> None:
        """Rows of `inp` (in_rows[d] of them to rank d, in rank order) into
        `out` (out_rows[s] from rank s, in rank order)."""
        dist.all_to_all_single(out, inp, [int(v) for v in out_rows], [int(v) for v in in_rows], group=self.group)


class ExpertParallelMoE:
    """One MoE layer of fixed (T, E, k, H, I) on one rank of an expert-parallel
    group.  `pool` and `slot_table` hold this rank's experts only:
    slot_table[j] is the slot of expert owned_experts(E, G, rank)[j].
    `exchange` carries the rows between ranks (DistExchange by default)."""

    def __init__(self, T: int, E: int, k: int, H: int, I: int, exchange=None,
                 mode: int = _lib.FT_ROUTE_SOFTMAX_RENORM, device="cuda"):
        self.exchange = exchange if exchange is not None else DistExchange()
        self.G = self.exchange.world_size
        self.rank = self.exchange.rank
        self.experts = owned_experts(E, self.G, self.rank)
        self.T, self.E, self.k, self.H, self.I = T, E, k, H, I
        self.E_local = E // self.G
        self.device = torch.device(device)
        self.layer = MoELayer(T, E, k, H, I, mode, device)
        self.x_send = torch.empty((T * k, H), dtype=torch.bfloat16, device=self.device)
        self.ffn_ws = torch.empty(256, dtype=torch.uint8, device=self.device)
        self.plan: Optional[ExchangePlan] = None
        self._pin: Optional[torch.Tensor] = None    # page-locked staging of the plan's index arrays
        self._idx: Optional[torch.Tensor] = None
        # ordering of the two staging buffers across calls, whatever streams the calls use:
        # the host rewrites _pin only after the previous copy out of it has run, and the copy
        # into _idx waits until the previous step's kernels have stopped reading _idx
        self._pin_copied: Optional[torch.cuda.Event] = None
        self._idx_free: Optional[torch.cuda.Event] = None

    def _workspace(self, n_recv: int) -> torch.Tensor:
        need = _lib.ffn_workspace_size(n_recv, self.H, self.I, self.E_local, 1)
        if need > self.ffn_ws.numel():
            self.ffn_ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        return self.ffn_ws

    def forward(self, x: torch.Tensor, logits: torch.Tensor, slot_table: torch.Tensor, pool: ExpertPool,
                stream=None) -> torch.Tensor:
        """The layer for this rank's T tokens; returns y fp32 [T, H]."""
        L, k, H = self.layer, self.k, self.H
        assert x.dtype == torch.bfloat16 and x.shape == (self.T, H) and x.is_contiguous()
        assert logits.dtype == torch.float32 and logits.shape == (self.T, self.E) and logits.is_contiguous()
        assert slot_table.dtype == torch.int32 and slot_table.numel() == self.E_local
        if stream is not None and stream != torch.cuda.current_stream():
            with torch.cuda.stream(stream):     # the collectives follow the current stream
                return self.forward(x, logits, slot_table, pool)
        s = _stream(None)
        P = self.T * k
        L.route(logits)
        L.permute()
        _lib.gather_rows(x.data_ptr(), self.T, H * 2, L.perm_src.data_ptr(), k, P, self.x_send.data_ptr(), s)

        plan = self.plan = ExchangePlan(self.exchange.gather_offsets(L.offsets), self.G, self.E, self.rank)
        n = plan.n_recv
        dev = self.device
        # the plan's three index arrays: one page-locked buffer, one copy
        m, El = max(n, 1), self.E_local
        need = 2 * m + El + 1
        if self._pin_copied is not None:
            self._pin_copied.synchronize()
        if self._pin is None or self._pin.numel() < need:
            self._pin = torch.empty(need, dtype=torch.int32, pin_memory=True)
            self._idx = torch.empty(need, dtype=torch.int32, device=dev)
            self._idx_free = None
        hp = self._pin.numpy()
        hp[:m] = plan.perm_src_local
        hp[m:2 * m] = plan.ret_idx
        hp[2 * m:need] = plan.local_offsets
        if self._idx_free is not None:
            torch.cuda.current_stream().wait_event(self._idx_free)
        self._idx[:need].copy_(self._pin[:need], non_blocking=True)
        self._pin_copied = torch.cuda.Event()
        self._pin_copied.record()
        perm_src_local, ret_idx, local_offsets = self._idx[:m], self._idx[m:2 * m], self._idx[2 * m:need]

        x_recv = torch.empty((max(n, 1), H), dtype=torch.bfloat16, device=dev)
        self.exchange.rows(x_recv[:n], self.x_send, plan.recv_rows, plan.send_rows)

        out_local = torch.empty((max(n, 1), H), dtype=torch.float32, device=dev)
        out_send = torch.empty((max(n, 1), H), dtype=torch.float32, device=dev)
        if n > 0:
            ws = self._workspace(n)
            _lib.ffn_nvfp4(x_recv.data_ptr(), n, H, self.I, self.E_local, 1, perm_src_local.data_ptr(),
                           local_offsets.data_ptr(), slot_table.data_ptr(), pool.ptr, pool.layout,
                           out_local.data_ptr(), ws.data_ptr(), ws.numel(), s)
            _lib.gather_rows(out_local.data_ptr(), n, H * 4, ret_idx.data_ptr(), 1, n, out_send.data_ptr(), s)

        self._idx_free = torch.cuda.Event()
        self._idx_free.record()                 # after the last kernel that reads _idx
        self.exchange.rows(L.out_perm, out_send[:n], plan.send_rows, plan.recv_rows)
        L.combine()
        return L.y
