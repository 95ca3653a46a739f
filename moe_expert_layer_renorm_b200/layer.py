"""Python-side plumbing around the C ABI: device buffers (torch), streams,
the expert slot pool and the slot manager.

Every step of the layer runs in libftmoe.so; this module only allocates
memory with torch and forwards pointers (there is no fallback path).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _lib
from ._lib import FT_DOWN, FT_GATE, FT_UP


def _ptr(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(s: Optional[torch.cuda.Stream]) -> int:
    s = torch.cuda.current_stream() if s is None else s
    return s.cuda_stream


def untile(block: np.ndarray, N: int, width: int, row_bytes: int) -> np.ndarray:
    """Stage-tiled bytes [S][N][width] -> row-major [N, row_bytes] (the first
    row_bytes of each row's S * width bytes)."""
    S = block.size // (N * width)
    return np.ascontiguousarray(block.reshape(S, N, width).transpose(1, 0, 2).reshape(N, S * width)[:, :row_bytes])


class ExpertPool:
    """A device pool of expert slots (NVFP4, or MXFP4 with fmt=FT_SCALE_MXFP4),
    row-major or stage-tiled (tiled=True; see ft_tiled_slot_layout_init)."""

    def __init__(self, H: int, I: int, num_slots: int, device="cuda", fmt: int = _lib.FT_SCALE_NVFP4,
                 tiled: bool = False):
        self.H, self.I, self.num_slots, self.fmt, self.tiled = H, I, num_slots, fmt, tiled
        self.layout = _lib.slot_layout(H, I, num_slots, fmt, tiled)
        # the canonical row-major layout of the same format, for slots read back to the host
        self.rows_layout = _lib.slot_layout(H, I, num_slots, fmt)
        self.slot_bytes = int(self.layout.slot_bytes)
        self.buf = torch.zeros(num_slots * self.slot_bytes, dtype=torch.uint8, device=device)
        self._pack_ws = torch.zeros(256, dtype=torch.uint8, device=device)

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    def shape(self, mat: int):
        return (self.I, self.H) if mat in (FT_GATE, FT_UP) else (self.H, self.I)

    def pack_into(self, slot: int, mat: int, w: torch.Tensor, stream=None) -> None:
        """Quantise fp32 weights w [N, K] (on the device) into `slot`, in the pool's format and layout."""
        N, K = self.shape(mat)
        assert w.shape == (N, K) and w.dtype == torch.float32 and w.is_cuda and w.is_contiguous()
        base = self.ptr + slot * self.slot_bytes
        if self.tiled:
            _lib.pack_slot(w.data_ptr(), mat, self.layout, base, self._pack_ws.data_ptr(), _stream(stream))
            return
        L = self.layout
        pack = _lib.mxfp4_pack if self.fmt == _lib.FT_SCALE_MXFP4 else _lib.nvfp4_pack
        pack(w.data_ptr(), N, K, base + L.codes_off[mat], base + L.scales_off[mat], L.ld_scale[mat],
             base + L.global_off[mat], self._pack_ws.data_ptr(), _stream(stream))

    def slot_view(self, slot: int) -> torch.Tensor:
        return self.buf[slot * self.slot_bytes:(slot + 1) * self.slot_bytes]

    def tensor_bytes(self, slot: int, mat: int):
        """(codes uint8 [N, K/2], scales uint8 [N, ld], global fp32) of one tensor, on the host, row-major."""
        N, K = self.shape(mat)
        L = self.layout
        ld = L.ld_scale[mat]
        s = self.slot_view(slot)
        if self.tiled:
            S = (K + 255) // 256
            codes = untile(s[L.codes_off[mat]:L.codes_off[mat] + S * N * 128].cpu().numpy(), N, 128, K // 2)
            scales = untile(s[L.scales_off[mat]:L.scales_off[mat] + S * N * 16].cpu().numpy(), N, 16, ld)
        else:
            codes = s[L.codes_off[mat]:L.codes_off[mat] + N * K // 2].view(N, K // 2).cpu().numpy()
            scales = s[L.scales_off[mat]:L.scales_off[mat] + N * ld].view(N, ld).cpu().numpy()
        g = s[L.global_off[mat]:L.global_off[mat] + 4].cpu().numpy().view("float32")[0]
        return codes, scales, float(g)

    def export_slot(self, slot: int) -> np.ndarray:
        """The slot as a host image in the row-major layout `rows_layout`
        (what the oracle and the host banks read)."""
        if not self.tiled:
            return self.slot_view(slot).cpu().numpy()
        R = self.rows_layout
        out = np.zeros(int(R.slot_bytes), np.uint8)
        for mat in range(3):
            c, sc, g = self.tensor_bytes(slot, mat)
            out[R.codes_off[mat]:R.codes_off[mat] + c.size] = c.reshape(-1)
            out[R.scales_off[mat]:R.scales_off[mat] + sc.size] = sc.reshape(-1)
            out[R.global_off[mat]:R.global_off[mat] + 4] = np.frombuffer(np.float32(g).tobytes(), np.uint8)
        return out


class MoELayer:
    """Buffers and calls for one MoE FFN layer of fixed (T, E, k, H, I)."""

    def __init__(self, T: int, E: int, k: int, H: int, I: int, mode: int = _lib.FT_ROUTE_SOFTMAX_RENORM,
                 device="cuda", fused_front: bool = False, whole: bool = False):
        self.T, self.E, self.k, self.H, self.I, self.mode = T, E, k, H, I, mode
        self.fused_front = fused_front   # route + permute through ft_moe_route_permute (separate calls only)
        # forward() through ft_moe_layer_nvfp4 (one launch for decode-sized batches); False: the four calls
        self.whole = whole and not fused_front
        P = T * k
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.ids = torch.empty((T, k), **i32)
        self.w = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.offsets = torch.empty(E + 1, **i32)
        self.perm_src = torch.empty(P, **i32)
        self.pair_to_row = torch.empty(P, **i32)
        self.out_perm = torch.empty((P, H), dtype=torch.float32, device=dev)
        self.y = torch.empty((T, H), dtype=torch.float32, device=dev)
        self.dev = dev
        self.perm_ws_bytes = _lib.permute_workspace_size(T, k, E)
        self.ffn_ws_bytes = _lib.ffn_workspace_size(T, H, I, E, k)
        self.layer_ws_bytes = _lib.layer_workspace_size(T, H, I, E, k)
        self._perm_ws = self._ffn_ws = self._layer_ws = None

    # workspaces, allocated on first use: the separate calls' (permute, ffn) and
    # the whole-layer call's, which is zero-filled once and left ready by every call
    @property
    def perm_ws(self) -> torch.Tensor:
        if self._perm_ws is None:
            self._perm_ws = torch.empty(max(self.perm_ws_bytes, 256), dtype=torch.uint8, device=self.dev)
        return self._perm_ws

    @property
    def ffn_ws(self) -> torch.Tensor:
        if self._ffn_ws is None:
            self._ffn_ws = torch.empty(max(self.ffn_ws_bytes, 256), dtype=torch.uint8, device=self.dev)
        return self._ffn_ws

    @property
    def layer_ws(self) -> torch.Tensor:
        if self._layer_ws is None:
            self._layer_ws = torch.zeros(max(self.layer_ws_bytes, 256), dtype=torch.uint8, device=self.dev)
        return self._layer_ws

    def route(self, logits: torch.Tensor, stream=None) -> None:
        _lib.route(logits.data_ptr(), self.T, self.E, self.k, self.mode, self.ids.data_ptr(), self.w.data_ptr(),
                   _stream(stream))

    def permute(self, stream=None) -> None:
        _lib.permute(self.ids.data_ptr(), self.T, self.k, self.E, self.offsets.data_ptr(), self.perm_src.data_ptr(),
                     self.pair_to_row.data_ptr(), self.perm_ws.data_ptr(), self.perm_ws_bytes, _stream(stream))

    def route_permute(self, logits: torch.Tensor, stream=None) -> None:
        _lib.route_permute(logits.data_ptr(), self.T, self.E, self.k, self.mode, self.ids.data_ptr(),
                           self.w.data_ptr(), self.offsets.data_ptr(), self.perm_src.data_ptr(),
                           self.pair_to_row.data_ptr(), self.perm_ws.data_ptr(), self.perm_ws_bytes, _stream(stream))

    def ffn(self, x: torch.Tensor, slot_table: torch.Tensor, pool: ExpertPool, stream=None) -> None:
        _lib.ffn_nvfp4(x.data_ptr(), self.T, self.H, self.I, self.E, self.k, self.perm_src.data_ptr(),
                       self.offsets.data_ptr(), slot_table.data_ptr(), pool.ptr, pool.layout,
                       self.out_perm.data_ptr(), self.ffn_ws.data_ptr(), self.ffn_ws_bytes, _stream(stream))

    def combine(self, stream=None) -> None:
        _lib.combine(self.out_perm.data_ptr(), self.pair_to_row.data_ptr(), self.w.data_ptr(), self.T, self.k,
                     self.H, self.y.data_ptr(), _stream(stream))

    def layer(self, x: torch.Tensor, logits: torch.Tensor, slot_table: torch.Tensor, pool: ExpertPool,
              stream=None) -> None:
        _lib.layer_nvfp4(x.data_ptr(), logits.data_ptr(), self.T, self.H, self.I, self.E, self.k, self.mode,
                         slot_table.data_ptr(), pool.ptr, pool.layout, self.ids.data_ptr(), self.w.data_ptr(),
                         self.offsets.data_ptr(), self.perm_src.data_ptr(), self.pair_to_row.data_ptr(),
                         self.out_perm.data_ptr(), self.y.data_ptr(), self.layer_ws.data_ptr(), self.layer_ws_bytes,
                         _stream(stream))

    def forward(self, x: torch.Tensor, logits: torch.Tensor, slot_table: torch.Tensor, pool: ExpertPool,
                stream=None) -> torch.Tensor:
        """route -> permute -> ffn -> combine, enqueued on one stream (one ft_moe_layer_nvfp4 call, or
        the four calls when the layer was made with whole=False)."""
        assert x.dtype == torch.bfloat16 and x.shape == (self.T, self.H) and x.is_contiguous()
        assert logits.dtype == torch.float32 and logits.shape == (self.T, self.E) and logits.is_contiguous()
        assert slot_table.dtype == torch.int32 and slot_table.numel() == self.E
        if self.whole:
            self.layer(x, logits, slot_table, pool, stream)
            return self.y
        if self.fused_front:
            self.route_permute(logits, stream)
        else:
            self.route(logits, stream)
            self.permute(stream)
        self.ffn(x, slot_table, pool, stream)
        self.combine(stream)
        return self.y


class SlotManager:
    """ctypes wrapper of the host LRU slot manager (ft_slot_*)."""

    def __init__(self, capacity: int, layout: _lib.SlotLayout, pool_ptr: int = 0, host_only: bool = False):
        h = ctypes.c_void_p()
        flags = _lib.FT_SLOT_HOST_ONLY if host_only else _lib.FT_SLOT_DEVICE
        _lib.check(_lib.lib().ft_slot_create(ctypes.byref(h), capacity, ctypes.byref(layout),
                                             ctypes.c_void_p(pool_ptr or None), flags))
        self.h = h
        self.layout = layout

    def register_host(self, layer: int, expert: int, src_ptr: int) -> None:
        _lib.check(_lib.lib().ft_slot_register_host(self.h, layer, expert, ctypes.c_void_p(src_ptr)))

    def acquire(self, layer: int, ids, table_ptr: int, table_len: int, compute=0, copy=0) -> None:
        arr = (ctypes.c_int32 * len(ids))(*[int(i) for i in ids])
        _lib.check(_lib.lib().ft_slot_acquire(self.h, layer, arr, len(ids), ctypes.c_void_p(table_ptr), table_len,
                                              ctypes.c_void_p(compute or None), ctypes.c_void_p(copy or None)))

    def inject_copy_failures(self, n: int) -> None:
        _lib.check(_lib.lib().ft_slot_inject_copy_failures(self.h, n))

    def stats(self) -> dict:
        s = _lib.SlotStats()
        _lib.check(_lib.lib().ft_slot_stats(self.h, ctypes.byref(s)))
        return {"hits": s.hits, "misses": s.misses, "evictions": s.evictions, "bytes_h2d": s.bytes_h2d,
                "copies": s.copies}

    def close(self) -> None:
        if self.h:
            _lib.lib().ft_slot_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
