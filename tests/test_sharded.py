"""The host side of the sharded-table gather, on CPU.

* engram_shard_rows and the route workspace size (host functions of the
  library: no kernel runs);
* the exchange of ShardedGather.gather_ids between two gloo ranks, each with
  its own ids and its own shard: the library's three device steps (route,
  serve, place) are replaced, inside the rank processes, by test doubles
  written with the oracle's hash and routing and plain numpy indexing, so
  that what is under test is the collective plumbing (split sizes, request
  and row order, byte transport).  The result must be the oracle's gather
  from the whole table on that rank's ids.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W
from oracle import engram_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("total", [1, 7, 97, 1 << 20])
@pytest.mark.parametrize("R", [1, 2, 3, 8, 64])
def test_shard_rows_split_the_table(total, R):
    table = np.arange(min(total, 1000))
    rows = [L.engram_shard_rows(total, R, r) for r in range(R)]
    assert sum(rows) == total
    if total <= 1000:
        assert rows == [len(O.shard_table(table[:, None], R, r)) for r in range(R)]
    with pytest.raises(ValueError):
        L.engram_shard_rows(total, R, R)


def test_route_workspace_holds_rows_and_block_counts():
    w = W.small_workload()
    cfg = L.make_config(w.orders, w.heads_per_order, w.row_dim, w.hidden, w.hc_mult, w.conv_kernel, w.dil,
                        w.pad_id, w.vocab, w.torch_dtype)
    n = w.B * w.T * w.nh
    blocks = -(-n // 256)
    need = L.engram_shard_route_workspace_size(cfg, w.B, w.T, 8)
    assert need >= 8 * n + 4 * 8 * blocks and need % 256 == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _doubles(w, p):
    """Oracle-based stand-ins for the three device steps (CPU tensors)."""
    offsets = np.asarray(p.offsets)

    def route(cfg, weights, ids, R, counts, req_rows, req_pos, ws, history=None, dev_status=None, stream=None):
        if ids.numel() == 0:
            counts.zero_()
            return
        idx = O.ngram_hash(ids.numpy(), w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
        c, rr, rp = O.shard_route((idx + offsets[None, None, :]).reshape(-1), R)
        counts.copy_(torch.from_numpy(c))
        req_rows.copy_(torch.from_numpy(rr))
        req_pos.copy_(torch.from_numpy(rp))

    def serve(cfg, shard, req_rows, out, dev_status=None, stream=None):
        out.copy_(shard[req_rows])

    def place(cfg, got, req_pos, e, n_e, dev_status=None, stream=None):
        if req_pos.numel() == 0:                 # as the library: nothing to place
            return
        e.view(n_e, -1)[req_pos.long()] = got

    return route, serve, place


def _rank_main(rank, world, port, out, empty_rank=-1):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    from hashed_gram_conditional_hash_b200 import sharded
    from hashed_gram_conditional_hash_b200 import _lib as Lr
    w = W.small_workload(B=2, T=50, orders=(2, 3, 4), seed=30 + rank)   # each rank its own ids
    p = W.make_params(w.replace(seed=30), "cpu")                          # one table for all ranks
    ids = W.make_params(w, "cpu").ids
    if rank == empty_rank:                                                  # no ids, still serves its shard
        ids = ids[:, :0].contiguous()
    Lr.engram_shard_route, Lr.engram_shard_serve, Lr.engram_shard_place = _doubles(w, p)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = Lr.make_config(w.orders, w.heads_per_order, w.row_dim, w.hidden, w.hc_mult, w.conv_kernel, w.dil,
                             w.pad_id, w.vocab, w.torch_dtype)
        full = p.table.numpy() if p.table.dtype != torch.bfloat16 else p.table.view(torch.int16).numpy()
        shard = torch.from_numpy(O.shard_table(full, world, rank))
        if p.table.dtype == torch.bfloat16:
            shard = shard.view(torch.bfloat16)
        sg = sharded.ShardedGather(cfg, shard, total_rows=p.table.shape[0], row_offsets=p.offsets,
                                   primes=p.primes, multipliers=p.mult)
        e = sg.gather_ids(ids)
        if ids.numel() == 0:
            out[rank] = e.shape[0] == 0, int(e.shape[0])
            return
        idx = O.ngram_hash(ids.numpy(), w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
        ref = O.gather(full, p.offsets, idx.reshape(-1, w.nh))
        got = e.view(torch.int16).numpy() if e.dtype == torch.bfloat16 else e.numpy()
        out[rank] = bool(np.array_equal(got, ref)), int(e.shape[0])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,empty_rank", [(2, -1), (3, -1), (2, 1)])
def test_sharded_gather_exchange_over_gloo_ranks(world, empty_rank):
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), out, empty_rank), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == list(range(world))
    for rank in range(world):
        ok, rows = res[rank]
        assert ok, "rank %d: e differs from the gather of the whole table" % rank
        assert rows == (0 if rank == empty_rank else 2 * 50)
