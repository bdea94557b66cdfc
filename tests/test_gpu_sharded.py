"""A table sharded over several devices (explainer §4.4: tables sharded across
GPUs, the touched rows collected with an All-to-All).

The route must list exactly the oracle's requests (owner = row mod R, local
row = row div R, grouped by shard, increasing row of e within a shard: bit
for bit), and route -> serve per shard -> place must rebuild the plain gather
of the whole table bit for bit.  One GPU holds every emulated shard here
(the exchanges become slices of one buffer); the NCCL path runs as a
one-rank group, and the two-rank exchange runs on gloo in test_sharded.py."""
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist

from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W
from hashed_gram_conditional_hash_b200.sharded import ShardedGather

from gpu_helpers import device_params, make_layer as _layer, oracle_ids
from oracle import engram_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"

ROUTE_CASES = [W.small_workload(), W.small_workload(B=2, T=130, orders=(2, 3, 4)),
               W.small_workload(B=1, T=1), W.small_workload(B=2, T=60, raw_vocab=6500),
               W.CONFIGS["model_bf16"], W.CONFIGS["large_table_bf16"]]


def _oracle_rows(p):
    w = p.w
    idx = O.ngram_hash(oracle_ids(p), w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
    return (idx + np.asarray(p.offsets)[None, None, :]).reshape(-1)


def _route(p, layer, R, ids=None, history=None, st=None):
    ids = p.ids if ids is None else ids
    B, T = ids.shape
    n = B * T * p.w.nh
    counts = torch.empty(R, dtype=torch.int64, device=DEV)
    req_rows = torch.empty(n, dtype=torch.int64, device=DEV)
    req_pos = torch.empty(n, dtype=torch.int32, device=DEV)
    ws = torch.empty(max(L.engram_shard_route_workspace_size(layer.cfg, B, T, R), 256), dtype=torch.uint8,
                     device=DEV)
    L.engram_shard_route(layer.cfg, layer.weights, ids, R, counts, req_rows, req_pos, ws, history, st)
    return counts, req_rows, req_pos


@pytest.mark.parametrize("R", [1, 2, 3, 8, 64])
@pytest.mark.parametrize("w", ROUTE_CASES, ids=[str(i) for i in range(len(ROUTE_CASES))])
def test_route_equals_oracle_requests(w, R):
    p = device_params(w)
    layer = _layer(p)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    counts, req_rows, req_pos = _route(p, layer, R, st=st)
    c, rr, rp = O.shard_route(_oracle_rows(p), R)
    assert L.engram_read_status(st) == 0
    np.testing.assert_array_equal(counts.cpu().numpy(), c)
    np.testing.assert_array_equal(req_rows.cpu().numpy(), rr)
    np.testing.assert_array_equal(req_pos.cpu().numpy(), rp)


@pytest.mark.parametrize("R", [2, 3, 8])
@pytest.mark.parametrize("w", [W.small_workload(), W.small_workload(B=2, T=130, orders=(2, 3, 4)),
                               W.small_workload(dtype="f32", B=2, T=50, row_dim=32, hidden=128, hc_mult=3),
                               W.CONFIGS["model_bf16"]], ids=["small", "orders234", "f32", "model"])
def test_emulated_shards_rebuild_the_plain_gather(w, R):
    p = device_params(w)
    layer = _layer(p)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    counts, req_rows, req_pos = _route(p, layer, R, st=st)
    n = req_rows.numel()
    got = torch.empty((n, w.row_dim), dtype=p.table.dtype, device=DEV)
    start = 0
    for r, c in enumerate(counts.tolist()):
        shard = p.table[r::R].contiguous()
        assert shard.shape[0] == L.engram_shard_rows(p.table.shape[0], R, r)
        L.engram_shard_serve(layer.cfg, shard, req_rows[start:start + c], got[start:start + c], st)
        start += c
    assert start == n
    e = torch.empty((w.B * w.T, w.nh * w.row_dim), dtype=p.table.dtype, device=DEV)
    L.engram_shard_place(layer.cfg, got, req_pos, e, n, st)
    assert L.engram_read_status(st) == 0
    assert torch.equal(e, layer.gather_ids(p.ids))


def test_route_with_history_continues_sequences():
    w = W.small_workload(B=3, T=40, orders=(2, 3, 4))
    p = device_params(w)
    layer = _layer(p)
    R = 3
    hist = p.ids[:, 17:20].contiguous()
    tail_ids = p.ids[:, 20:].contiguous()
    counts, req_rows, req_pos = _route(p, layer, R, ids=tail_ids, history=hist)
    # the tail's requests are the full sequence's requests at positions >= 20
    rows = _oracle_rows(p).reshape(w.B, w.T, w.nh)[:, 20:].reshape(-1)
    c, rr, rp = O.shard_route(rows, R)
    np.testing.assert_array_equal(counts.cpu().numpy(), c)
    np.testing.assert_array_equal(req_rows.cpu().numpy(), rr)
    np.testing.assert_array_equal(req_pos.cpu().numpy(), rp)


def test_serve_and_place_flag_out_of_range_rows():
    w = W.small_workload(B=1, T=8)
    p = device_params(w)
    layer = _layer(p)
    shard = p.table[0::2].contiguous()
    asked = torch.tensor([0, shard.shape[0], 5, -1], dtype=torch.int64, device=DEV)
    out = torch.full((4, w.row_dim), 7, dtype=p.table.dtype, device=DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.engram_shard_serve(layer.cfg, shard, asked, out, st)
    assert L.engram_read_status(st) == 2                 # ENGRAM_STATUS_ROW_RANGE
    assert torch.equal(out[0], shard[0]) and torch.equal(out[2], shard[5])
    assert not out[1].any() and not out[3].any()
    e = torch.zeros((2, w.row_dim), dtype=p.table.dtype, device=DEV)
    st.zero_()
    pos = torch.tensor([1, 2, -3, 0], dtype=torch.int32, device=DEV)
    L.engram_shard_place(layer.cfg, out, pos, e, 2, st)
    assert L.engram_read_status(st) == 2
    assert torch.equal(e[1], out[0]) and torch.equal(e[0], out[3])


def test_empty_batch_routes_nothing():
    w = W.small_workload(B=2, T=5)
    p = device_params(w)
    layer = _layer(p)
    counts = torch.full((4,), -1, dtype=torch.int64, device=DEV)
    ids = torch.empty((2, 0), dtype=torch.int64, device=DEV)
    empty64 = torch.empty(0, dtype=torch.int64, device=DEV)
    L.engram_shard_route(layer.cfg, layer.weights, ids, 4, counts, empty64,
                         torch.empty(0, dtype=torch.int32, device=DEV), torch.empty(256, dtype=torch.uint8, device=DEV))
    assert counts.tolist() == [0, 0, 0, 0]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_sharded_gather_one_rank_nccl_group_then_forward():
    w = W.small_workload(B=2, T=130, orders=(2, 3, 4))
    p = device_params(w)
    layer = _layer(p)
    store = dist.TCPStore("127.0.0.1", _free_port(), 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=torch.device(DEV, 0),
                            timeout=timedelta(seconds=60))
    try:
        sg = ShardedGather(layer.cfg, p.table, total_rows=p.table.shape[0], row_offsets=p.offsets,
                           primes=p.primes, multipliers=p.mult, lookup=p.lookup)
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        e = sg.gather_ids(p.ids, dev_status=st)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert L.engram_read_status(st) == 0
    assert torch.equal(e, layer.gather_ids(p.ids))
    assert torch.equal(layer.forward_gathered(e, p.hidden), layer.forward(p.ids, p.hidden))
