"""One Engram layer's table sharded over the ranks of a process group.

The explainer page (§4.4, system efficiency) shards the embedding tables
across GPUs in training and collects the rows a batch touches with an
All-to-All.  Shard r of R holds the stacked table's rows r, r+R, r+2R, ...
(the split libengram's engram_shard_* calls use).  The gather of e for this
rank's ids runs as

  engram_shard_route   this rank's ids -> requests grouped by owner shard
  all-to-all           request counts, then the requested local rows
  engram_shard_serve   the rows the other ranks asked of this rank's shard
  all-to-all           the rows back, in request order
  engram_shard_place   received rows -> their rows of e

and e equals the gather from the whole table bit for bit; the rest of the
pass runs on it through engram_forward_gathered.  Every step on the rows runs
in libengram's kernels; the exchanges are torch.distributed collectives (NCCL
over NVLink on GPUs), moved as bytes so that any table dtype travels
unchanged.  The split sizes of the second and third exchange are the counts
of the first, read back to the host (all_to_all_single takes them as lists).
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

from . import _lib as L


class ShardedGather:
    """This rank's shard of one layer's table and the hash parameters of the
    whole table (row offsets, primes and multipliers of every head, the total
    row count)."""

    def __init__(self, cfg: L.EngramConfig, shard: torch.Tensor, *, total_rows: int, row_offsets, primes,
                 multipliers, lookup: Optional[torch.Tensor] = None, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        if self.world > L.MAX_SHARDS:
            raise ValueError("at most %d shards" % L.MAX_SHARDS)
        if shard.shape[0] != L.engram_shard_rows(total_rows, self.world, self.rank):
            raise ValueError("shard %d of %d must hold %d rows, not %d" % (
                self.rank, self.world, L.engram_shard_rows(total_rows, self.world, self.rank), shard.shape[0]))
        if not shard.is_contiguous():
            raise ValueError("the shard must be contiguous")
        self.cfg = cfg
        self.shard = shard
        self.nh = cfg.n_orders * cfg.heads_per_order
        self.row_width = shard.shape[1]
        self._host = [np.ascontiguousarray(np.asarray(a, dtype=np.int64)) for a in (row_offsets, primes, multipliers)]
        self._lookup = lookup
        w = L.EngramWeights()
        w.table = shard.data_ptr()           # not read by the route
        w.total_rows = int(total_rows)
        w.row_offsets = self._host[0].ctypes.data
        w.primes = self._host[1].ctypes.data
        w.multipliers = self._host[2].ctypes.data
        w.lookup = lookup.data_ptr() if lookup is not None else None
        w.raw_vocab = lookup.numel() if lookup is not None else 0
        self.weights = w

    def route(self, ids: torch.Tensor, history: Optional[torch.Tensor] = None,
              dev_status: Optional[torch.Tensor] = None, stream=None):
        """(counts [R], req_rows [N], req_pos [N]) of engram_shard_route."""
        B, T = ids.shape
        n = B * T * self.nh
        dev = ids.device
        counts = torch.empty(self.world, dtype=torch.int64, device=dev)
        req_rows = torch.empty(n, dtype=torch.int64, device=dev)
        req_pos = torch.empty(n, dtype=torch.int32, device=dev)
        ws = torch.empty(max(L.engram_shard_route_workspace_size(self.cfg, B, T, self.world), 256),
                         dtype=torch.uint8, device=dev)
        L.engram_shard_route(self.cfg, self.weights, ids, self.world, counts, req_rows, req_pos, ws, history,
                             dev_status, stream)
        return counts, req_rows, req_pos

    def gather_ids(self, ids: torch.Tensor, e: Optional[torch.Tensor] = None,
                   history: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
        """e [B*T, nh*Dh] of this rank's ids; every rank of the group calls it
        (collectively, in the same order), each with its own ids."""
        B, T = ids.shape
        n = B * T * self.nh
        dev = ids.device
        counts, req_rows, req_pos = self.route(ids, history, dev_status)
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts, group=self.group)
        send = counts.tolist()
        recv = recv_counts.tolist()
        asked = torch.empty(sum(recv), dtype=torch.int64, device=dev)
        dist.all_to_all_single(asked, req_rows, recv, send, group=self.group)
        served = torch.empty((sum(recv), self.row_width), dtype=self.shard.dtype, device=dev)
        L.engram_shard_serve(self.cfg, self.shard, asked, served, dev_status)
        got = torch.empty((n, self.row_width), dtype=self.shard.dtype, device=dev)
        dist.all_to_all_single(got.view(torch.uint8), served.view(torch.uint8), send, recv, group=self.group)
        if e is None:
            e = torch.empty((B * T, self.nh * self.row_width), dtype=self.shard.dtype, device=dev)
        L.engram_shard_place(self.cfg, got, req_pos, e, n, dev_status)
        return e
