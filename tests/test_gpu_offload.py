"""The pass in two halves (engram_gather_ids, then engram_forward_gathered)
and tables resident in pinned host memory (explainer §4.4: the indices depend
only on the ids, so rows can be fetched ahead of the layer, from host RAM).

The halves must give engram_forward's result bit for bit, and a host-resident
table the device-resident result bit for bit (the same rows reach the same
kernels); pageable host memory is refused without a launch."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_hash_b200 import EngramLayer
from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W

from gpu_helpers import device_params, make_layer, oracle_ids
from oracle import engram_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(p, table=None):
    return make_layer(p, table)


CASES = [W.small_workload(), W.small_workload(B=2, T=130, hidden=512, hc_mult=4, orders=(2, 3, 4)),
         W.small_workload(B=2, T=60, raw_vocab=6500), W.small_workload(dtype="f32", B=2, T=50, row_dim=32,
                                                                       hidden=128, hc_mult=3),
         W.CONFIGS["model_bf16"]]


@pytest.mark.parametrize("w", CASES, ids=[str(i) for i in range(len(CASES))])
def test_gathered_halves_equal_forward(w):
    p = device_params(w)
    layer = _layer(p)
    y = layer.forward(p.ids, p.hidden)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    e = layer.gather_ids(p.ids, dev_status=st)
    y2 = layer.forward_gathered(e, p.hidden, dev_status=st)
    assert L.engram_read_status(st) == 0
    assert torch.equal(y, y2)
    # the rows are the table rows at the oracle's indices
    idx = O.ngram_hash(oracle_ids(p), w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
    rows = torch.from_numpy(idx + np.asarray(p.offsets)[None, None, :]).to(DEV).view(-1)
    assert torch.equal(e, p.table[rows].view(e.shape))


@pytest.mark.parametrize("w", CASES, ids=[str(i) for i in range(len(CASES))])
def test_host_resident_table_equals_device_table(w):
    p = device_params(w)
    dev_layer = _layer(p)
    host_layer = _layer(p, table=p.table.cpu().pin_memory())
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    assert torch.equal(host_layer.gather_ids(p.ids, dev_status=st), dev_layer.gather_ids(p.ids))
    assert torch.equal(host_layer.forward(p.ids, p.hidden, dev_status=st), dev_layer.forward(p.ids, p.hidden))
    assert L.engram_read_status(st) == 0


def test_gather_ids_with_history_continues_sequences():
    w = W.small_workload(B=3, T=40, orders=(2, 3, 4))
    p = device_params(w)
    layer = _layer(p)
    full = layer.gather_ids(p.ids)
    hist = p.ids[:, 17:20].contiguous()               # the 3 ids before position 20
    tail = layer.gather_ids(p.ids[:, 20:].contiguous(), history=hist)
    E = w.nh * w.row_dim
    assert torch.equal(tail.view(w.B, -1, E), full.view(w.B, w.T, E)[:, 20:])


def test_pageable_host_table_is_refused_without_launch():
    w = W.small_workload()
    p = device_params(w)
    with pytest.raises(ValueError):
        _layer(p, table=p.table.cpu())                 # the binding refuses it up front
    layer = _layer(p)
    pageable = p.table.cpu()                          # ... and so does the library itself
    layer.weights.table = pageable.data_ptr()
    e = torch.empty((w.B * w.T, w.nh * w.row_dim), dtype=p.table.dtype, device=DEV)
    before = L.engram_launch_count()
    with pytest.raises(L.EngramError) as ei:
        L.engram_gather_ids(layer.cfg, layer.weights, p.ids, e)
    assert ei.value.code == 1 and "pinned" in str(ei.value)
    with pytest.raises(L.EngramError):
        layer.forward(p.ids, p.hidden)
    assert L.engram_launch_count() == before


def _oracle_rows(p, x, hist=None):
    """Each row of e as the oracle gives it: the table row at the oracle's
    index (its own multipliers and primes), for a table on the device or in
    pinned host memory."""
    w = p.w
    idx = O.ngram_hash(x, w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id, hist=hist)
    rows = torch.from_numpy((idx + np.asarray(p.offsets)[None, None, :]).reshape(-1))
    return p.table[rows.to(p.table.device)].reshape(x.shape[0] * x.shape[1], w.nh * w.row_dim).cpu()


GATHER_SHAPES = [
    dict(B=3, T=5, orders=(2, 3), heads_per_order=1),              # 2 heads: a warp spans many short sequences
    dict(B=4, T=7, orders=(2, 3, 4), heads_per_order=1),           # 3 heads (odd), rows cross tokens mid-warp
    dict(B=2, T=33, orders=(2,), heads_per_order=1),               # 1 head: the 16-row form
    dict(B=2, T=19, orders=(1, 2, 3, 4, 5, 6, 7, 8), heads_per_order=8, vocab=3000),  # 64 heads, order 8
    dict(B=5, T=61, orders=(2, 3, 4), heads_per_order=5),          # 15 heads
    dict(B=1, T=1),                                                # a single token
]


@pytest.mark.parametrize("kw", GATHER_SHAPES, ids=[str(i) for i in range(len(GATHER_SHAPES))])
@pytest.mark.parametrize("with_history", [False, True])
def test_gather_ids_bit_exact_against_oracle(kw, with_history):
    # the hash + gather kernel's rows, bit for bit, over shapes that put the
    # edges of sequences and tokens at every place inside a warp's rows
    w = W.small_workload(prime_base=1009, **kw)
    p = device_params(w)
    layer = _layer(p)
    x = oracle_ids(p)
    hist = None
    if with_history:
        g = np.random.default_rng(5)
        hist = torch.from_numpy(g.integers(0, w.vocab, size=(w.B, w.max_n - 1))).to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    e = layer.gather_ids(p.ids, history=hist, dev_status=st)
    assert L.engram_read_status(st) == 0
    expect = _oracle_rows(p, x, hist=None if hist is None else hist.cpu().numpy())
    assert torch.equal(e.cpu(), expect)
    # e 16 bytes off a 32-byte boundary takes the 16-byte form: same rows
    buf = torch.empty(e.numel() * e.element_size() + 64, dtype=torch.uint8, device=DEV)
    off = (16 - buf.data_ptr() % 32) % 32
    e16 = buf[off: off + e.numel() * e.element_size()].view(e.dtype).view(e.shape)
    assert e16.data_ptr() % 32 == 16
    layer.gather_ids(p.ids, e=e16, history=hist)
    assert torch.equal(e16.cpu(), expect)


def test_gather_ids_layers_equals_per_layer_gathers():
    # two Engram layers of one model (the pages' layers 2 and 6): own
    # multipliers and tables, the same ids; one host-resident table
    base = W.small_workload(B=3, T=90, orders=(2, 3, 4), heads_per_order=3)
    ws_ = [base.replace(layer_id=2, seed=21), base.replace(layer_id=6, seed=22)]
    ps = [device_params(w) for w in ws_]
    ps[1].table = ps[1].table.cpu().pin_memory()
    layers = [_layer(p) for p in ps]
    ids = ps[0].ids
    assert not np.array_equal(ps[0].mult, ps[1].mult)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    e = [torch.empty((base.B * base.T, base.nh * base.row_dim), dtype=ps[0].table.dtype, device=DEV)
         for _ in layers]
    L.engram_gather_ids_layers(layers[0].cfg, [l.weights for l in layers], ids, e, dev_status=st)
    assert L.engram_read_status(st) == 0
    x = oracle_ids(ps[0])
    for p_l, layer, e_l in zip(ps, layers, e):
        assert torch.equal(e_l, layer.gather_ids(ids))
        # every layer's rows, bit for bit, from the oracle's hash with that
        # layer's multipliers and primes and that layer's table
        assert torch.equal(e_l.cpu(), _oracle_rows(p_l, x))
    # and the rows reach each layer's own forward
    y0 = layers[0].forward_gathered(e[0], ps[0].hidden)
    assert torch.equal(y0, layers[0].forward(ids, ps[0].hidden))


def test_gather_ids_layers_with_history_continues_sequences():
    base = W.small_workload(B=3, T=40, orders=(2, 3, 4))
    ps = [device_params(base.replace(layer_id=1, seed=31)), device_params(base.replace(layer_id=4, seed=32))]
    layers = [_layer(p) for p in ps]
    ids = ps[0].ids
    hist = ids[:, 17:20].contiguous()                 # the 3 ids before position 20
    tail = ids[:, 20:].contiguous()
    E = base.nh * base.row_dim
    e = [torch.empty((base.B * 20, E), dtype=ps[0].table.dtype, device=DEV) for _ in layers]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.engram_gather_ids_layers(layers[0].cfg, [l.weights for l in layers], tail, e, history=hist, dev_status=st)
    assert L.engram_read_status(st) == 0
    x = ids.cpu().numpy()
    for p_l, layer, e_l in zip(ps, layers, e):
        full = layer.gather_ids(ids)
        assert torch.equal(e_l.view(base.B, -1, E), full.view(base.B, base.T, E)[:, 20:])
        # the oracle's hash of the tail with the same history
        assert torch.equal(e_l.cpu(), _oracle_rows(p_l, x[:, 20:], hist=x[:, 17:20]))
