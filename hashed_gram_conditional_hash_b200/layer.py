"""Convenience wrapper that binds one Engram layer's parameters to libengram.

It holds the C structs (config, weights), keeps the host parameter arrays
alive for the library, allocates workspaces and streaming states with torch,
and forwards to the C entry points.  No arithmetic of the method happens here.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from . import _lib as L


@dataclass
class StreamState:
    """Device buffers of an engram_state plus the C struct that points at them."""
    c: L.EngramState
    id_ring: torch.Tensor
    v_ring: torch.Tensor
    g_ring: torch.Tensor
    pos: torch.Tensor


class EngramLayer:
    def __init__(self, *, orders, heads_per_order, row_dim, hidden, hc_mult, conv_kernel,
                 dilation, pad_id, vocab, table, row_offsets, primes, multipliers, w_value,
                 w_key, norm_key, norm_query, conv_w, lookup=None, rms_eps=1e-6, gate_eps=1e-6):
        self.dtype = table.dtype
        self.cfg = L.make_config(orders, heads_per_order, row_dim, hidden, hc_mult, conv_kernel,
                                 dilation, pad_id, vocab, table.dtype, rms_eps, gate_eps)
        self.max_n = max(orders)
        self.hidden, self.hc = hidden, hc_mult
        self.ring_len = (conv_kernel - 1) * dilation + 1
        self._host = [np.ascontiguousarray(np.asarray(a, dtype=np.int64))
                      for a in (row_offsets, primes, multipliers)]
        self._dev = [table, w_value, w_key, norm_key, norm_query, conv_w, lookup]
        # the table may live in pinned host memory (read over the host link);
        # everything else, and every workspace, lives on the weights' device
        self.device = w_value.device
        if table.device.type == "cpu" and not table.is_pinned():
            raise ValueError("a host-resident table must be in pinned memory (tensor.pin_memory())")
        self.row_width = table.shape[1]
        self.nh = len(primes)
        for t in self._dev:
            if t is not None and not t.is_contiguous():
                raise ValueError("layer tensors must be contiguous")
        w = L.EngramWeights()
        w.table = table.data_ptr()
        w.total_rows = table.shape[0]
        w.row_offsets = self._host[0].ctypes.data
        w.primes = self._host[1].ctypes.data
        w.multipliers = self._host[2].ctypes.data
        w.lookup = lookup.data_ptr() if lookup is not None else None
        w.raw_vocab = lookup.numel() if lookup is not None else 0
        w.w_value = w_value.data_ptr()
        w.w_key = w_key.data_ptr()
        w.norm_key = norm_key.data_ptr()
        w.norm_query = norm_query.data_ptr()
        w.conv_w = conv_w.data_ptr()
        self.weights = w

    @classmethod
    def from_params(cls, p) -> "EngramLayer":
        """From a workloads.Params whose tensors are on a CUDA device."""
        w = p.w
        return cls(orders=w.orders, heads_per_order=w.heads_per_order, row_dim=w.row_dim,
                   hidden=w.hidden, hc_mult=w.hc_mult, conv_kernel=w.conv_kernel,
                   dilation=w.dil, pad_id=w.pad_id, vocab=w.vocab, table=p.table,
                   row_offsets=p.offsets, primes=p.primes, multipliers=p.mult,
                   w_value=p.w_value, w_key=p.w_key, norm_key=p.norm_key,
                   norm_query=p.norm_query, conv_w=p.conv_w, lookup=p.lookup,
                   rms_eps=w.rms_eps, gate_eps=w.gate_eps)

    def workspace(self, B: int, T: int, device=None) -> torch.Tensor:
        n = L.engram_forward_workspace_size(self.cfg, B, T)
        return torch.empty(max(n, 256), dtype=torch.uint8,
                           device=device or self.device)

    def new_state(self, B: int, stream=None) -> StreamState:
        dev = self.device
        id_ring = torch.empty((B, max(self.max_n - 1, 1)), dtype=torch.int64, device=dev)
        v_ring = torch.empty((B, self.ring_len, self.hidden), dtype=self.dtype, device=dev)
        g_ring = torch.empty((B, self.ring_len, self.hc), dtype=torch.float32, device=dev)
        pos = torch.empty((B,), dtype=torch.int64, device=dev)
        c = L.EngramState()
        c.id_ring = id_ring.data_ptr()
        c.v_ring = v_ring.data_ptr()
        c.g_ring = g_ring.data_ptr()
        c.pos = pos.data_ptr()
        c.ring_len = self.ring_len
        L.engram_state_init(self.cfg, c, B, stream)
        return StreamState(c, id_ring, v_ring, g_ring, pos)

    def gather_ids(self, ids: torch.Tensor, e: Optional[torch.Tensor] = None,
                   history: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                   stream=None) -> torch.Tensor:
        """The gathered rows e [B*T, nh*Dh] of ids (engram_gather_ids)."""
        B, T = ids.shape
        if e is None:
            e = torch.empty((B * T, self.nh * self.row_width), dtype=self.dtype, device=ids.device)
        L.engram_gather_ids(self.cfg, self.weights, ids, e, history, dev_status, stream)
        return e

    def forward_gathered(self, e: torch.Tensor, hidden: torch.Tensor, y: Optional[torch.Tensor] = None,
                         ws: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
        """The pass on rows from gather_ids (engram_forward_gathered), no state."""
        B, T = hidden.shape[0], hidden.shape[1]
        if y is None:
            y = torch.empty((B, T, self.hc, self.hidden), dtype=self.dtype, device=hidden.device)
        if ws is None:
            ws = self.workspace(B, T, hidden.device)
        L.engram_forward_gathered(self.cfg, self.weights, e, B, T, hidden, y, ws, dev_status, stream)
        return y

    def forward(self, ids: torch.Tensor, hidden: torch.Tensor, y: Optional[torch.Tensor] = None,
                ws: Optional[torch.Tensor] = None, state: Optional[StreamState] = None,
                dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        B, T = ids.shape
        if y is None:
            y = torch.empty((B, T, self.hc, self.hidden), dtype=self.dtype, device=ids.device)
        if ws is None:
            ws = self.workspace(B, T, ids.device)
        L.engram_forward(self.cfg, self.weights, ids, hidden, y, ws,
                         state.c if state is not None else None, dev_status, stream)
        return y
