"""GPU parity of engram_forward (the whole pass through the C ABI) against the
float64 oracle: full comparison on few-tile shapes with ragged tails, sampled
positions (sequence edges + random interior) on the full-size workloads in
the launch configuration the benchmark times, plus degenerate cases."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_hash_b200 import EngramLayer
from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W

from gpu_helpers import (TOL, device_params, oracle_at, oracle_forward_full, oracle_ids, rel_err,
                         sample_positions)
from oracle import engram_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"


ENGINE_FLAGS = {"auto": 0, "simt": L.DEBUG_FORCE_SIMT, "fused": L.DEBUG_FUSED_GATHER,
                "simt_fused": L.DEBUG_FORCE_SIMT | L.DEBUG_FUSED_GATHER,
                "single_cta": L.DEBUG_TC_SINGLE_CTA, "mblock_order": L.DEBUG_TILE_MBLOCK_ORDER}


def _run(p, engine="auto", conv_w=None, chunks=1):
    L.engram_set_debug(ENGINE_FLAGS[engine])
    L.engram_set_overlap_chunks(chunks)
    try:
        layer = EngramLayer.from_params(p)
        if conv_w is not None:
            layer.weights.conv_w = conv_w.data_ptr()
        st = torch.zeros(1, dtype=torch.int32, device=DEV)
        y = layer.forward(p.ids, p.hidden, dev_status=st)
        assert L.engram_read_status(st) == 0
        return y
    finally:
        L.engram_set_debug(0)
        L.engram_set_overlap_chunks(0)


SMALL = [
    dict(),                                                        # bf16, B=3, T=77, hc=2
    dict(B=2, T=130, hidden=512, hc_mult=4, orders=(2, 3, 4), dilation=4),
    dict(B=1, T=1),
    dict(B=4, T=3, hc_mult=1),
    dict(dtype="f32", B=2, T=50, row_dim=32, hidden=128, hc_mult=3),
    dict(B=2, T=200, heads_per_order=4, hidden=768, hc_mult=2),   # 768 = 3 tiles of 256
    dict(B=2, T=70, conv_kernel=6, dilation=2),                   # generic tap count
    dict(B=1, T=150, dilation=9, hc_mult=3),                      # long halo (R = 27)
    dict(B=2, T=45, row_dim=20),                                  # 40-byte rows
    dict(B=2, T=90, hc_mult=6, hidden=128),                       # more than 4 branches
    dict(B=2, T=60, raw_vocab=6500),                              # raw ids through the lookup
    dict(B=2, T=41, row_dim=32),                                  # 64-byte rows (generic gather)
    dict(B=1, T=37, row_dim=128, orders=(2, 3, 4)),               # 256-byte rows (generic gather)
    dict(B=2, T=33, orders=(2,), heads_per_order=1),               # one head in all (16-row gather)
    dict(B=2, T=40, orders=(1, 8), dilation=8),                    # a unigram and the largest order
]


@pytest.mark.parametrize("kw", SMALL, ids=[str(i) for i in range(len(SMALL))])
@pytest.mark.parametrize("engine", ["auto", "simt", "fused", "simt_fused", "single_cta"])
def test_forward_small_full(kw, engine):
    w = W.small_workload(**kw)
    p = device_params(w)
    y = _run(p, engine)
    ref = oracle_forward_full(p)
    assert rel_err(y.double().cpu().numpy(), ref["Y"]) <= TOL[w.dtype]


def test_forward_tiny_f32_full():
    w = W.CONFIGS["tiny_f32"]
    p = device_params(w)
    y = _run(p)
    ref = oracle_forward_full(p)
    err = rel_err(y.double().cpu().numpy(), ref["Y"])
    assert err <= TOL["f32"], err


@pytest.mark.parametrize("name", ["model_bf16", "model_bf16_norm_w", "large_table_bf16", "hbm_table_bf16"])
def test_forward_full_size_sampled(name):
    # the bench's launch configuration at full size: both tensor-core engines
    # against the oracle at the sequence edges plus 4096 random positions;
    # "_norm_w": RMSNorm weights 1 + N(0, 0.1^2) instead of exactly 1, so the
    # weight products of the key epilogue are exercised at full size
    if name.endswith("_norm_w"):
        w = W.CONFIGS[name[: -len("_norm_w")]].replace(norm_w_std=0.1)
    else:
        w = W.CONFIGS[name]
    p = device_params(w)
    pos = sample_positions(w.B, w.T, w.dil, 4096, seed=11)
    Yref, _, _, _ = oracle_at(p, pos)
    bi = torch.tensor([b for b, _ in pos], device=DEV)
    ti = torch.tensor([t for _, t in pos], device=DEV)
    for engine, chunks in (("auto", 1), ("single_cta", 1), ("auto", 4)):
        y = _run(p, engine, chunks=chunks)
        err = rel_err(y[bi, ti].double().cpu().numpy(), Yref)
        assert err <= TOL[w.dtype], (engine, chunks, err)
        del y


@pytest.mark.parametrize("name", ["tiny_f32", "model_bf16", "large_table_bf16", "hbm_table_bf16"])
def test_gathered_rows_full_size_bit_exact(name):
    # white-box: on the gather-then-project path the forward's workspace starts
    # with e [M, E]; every row must be the table row at the oracle's index
    w = W.CONFIGS[name]
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    ws = layer.workspace(w.B, w.T)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    layer.forward(p.ids, p.hidden, ws=ws, dev_status=st)
    assert L.engram_read_status(st) == 0
    idx = O.ngram_hash(oracle_ids(p), w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
    rows = torch.from_numpy(idx + np.asarray(p.offsets)[None, None, :]).to(DEV).view(-1)
    M, E = w.B * w.T, w.nh * w.row_dim
    expect = p.table[rows].view(M, E)
    e = ws[: M * E * p.table.element_size()].view(p.table.dtype).view(M, E)
    assert torch.equal(e, expect)


def test_forward_zero_conv_is_gated_value():
    w = W.small_workload(B=2, T=40)
    p = device_params(w)
    zero = torch.zeros_like(p.conv_w)
    y = _run(p, conv_w=zero)
    ref = oracle_forward_full(p, conv_w=zero)
    assert rel_err(y.double().cpu().numpy(), ref["g"][..., None] * ref["V"][:, :, None, :]) <= TOL["bf16"]


def test_forward_branch_with_zero_hidden_gates_one_half():
    # a branch whose hidden state is zero has s = 0, so g = 1/2 exactly
    # (formulas page §2.2 step 2) and its Y is the conv of V/2
    w = W.small_workload(B=2, T=100, hidden=512, hc_mult=4)
    p = device_params(w)
    p.hidden[:, :, 2] = 0
    ref = oracle_forward_full(p)
    assert np.all(ref["s"][:, :, 2] == 0.0) and np.all(ref["g"][:, :, 2] == 0.5)
    for engine in ("auto", "simt"):
        y = _run(p, engine)
        assert rel_err(y.double().cpu().numpy(), ref["Y"]) <= TOL["bf16"], engine


OVERLAP = [
    (dict(B=2, T=300, hidden=512, hc_mult=4), 2),
    (dict(B=5, T=130, hidden=256, hc_mult=2, orders=(2, 3, 4), dilation=4), 3),  # uneven chunks
    (dict(B=3, T=77), 8),                                                         # clipped to B
    (dict(B=4, T=40, hidden=768, hc_mult=3, dilation=9), 2),                     # long halo, short chunks
]


@pytest.mark.parametrize("kw,chunks", OVERLAP, ids=[str(i) for i in range(len(OVERLAP))])
def test_forward_overlapped_chunks_equal_plain(kw, chunks):
    # the pass in sequence chunks whose gate and conv overlap the next chunk's
    # projection on two streams: the same kernels per element, so the same bits
    w = W.small_workload(**kw)
    p = device_params(w)
    plain = _run(p, chunks=1)
    y = _run(p, chunks=chunks)
    assert torch.equal(y, plain)
    assert rel_err(y.double().cpu().numpy(), oracle_forward_full(p)["Y"]) <= TOL[w.dtype]


def test_forward_overlapped_chunks_model_shaped():
    w = W.CONFIGS["model_bf16"]
    p = device_params(w)
    plain = _run(p, chunks=1)
    for chunks in (2, 4):
        assert torch.equal(_run(p, chunks=chunks), plain), chunks


def test_forward_split_value_tail_tiles():
    # 2 M-blocks x 40 column tiles = 80 pair tiles: the 6 left for a last
    # round of pairs run as 12 half-width value tiles
    w = W.small_workload(B=2, T=256, hidden=2048, hc_mult=4)
    p = device_params(w)
    y = _run(p, "auto")
    ref = oracle_forward_full(p)
    assert rel_err(y.double().cpu().numpy(), ref["Y"]) <= TOL[w.dtype]
    # the same rows through the single-CTA engine (no tile split)
    d = _run(p, "single_cta").double()
    assert (y.double() - d).abs().max().item() <= 1e-2 * d.abs().max().item()


@pytest.mark.parametrize("kw", [dict(B=2, T=256, hidden=2048, hc_mult=4),   # split value tail
                                dict(B=4, T=300, hidden=512, hc_mult=4),    # several groups of M-blocks
                                dict(B=3, T=77)])
def test_forward_tile_orders_agree(kw):
    # the projection's tiles in groups of M-blocks (default) or M-block by
    # M-block: every output element is the same computation, so the same bits
    w = W.small_workload(**kw)
    p = device_params(w)
    assert torch.equal(_run(p), _run(p, "mblock_order"))


def test_forward_engines_agree():
    w = W.small_workload(B=2, T=300, hidden=512, hc_mult=4)
    p = device_params(w)
    a = _run(p, "auto").double()
    b = _run(p, "simt").double()
    c = _run(p, "fused").double()
    d = _run(p, "single_cta").double()
    assert (a - b).abs().max().item() <= 2e-2 * b.abs().max().item()
    # the fused gather feeds the same rows to the single-CTA MMA: identical results
    assert torch.equal(c, d)
    assert (a - d).abs().max().item() <= 1e-2 * d.abs().max().item()


def test_forward_empty_is_noop():
    w = W.small_workload()
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    ids = torch.empty((0, 5), dtype=torch.int64, device=DEV)
    hid = torch.empty((0, 5, w.hc_mult, w.hidden), dtype=w.torch_dtype, device=DEV)
    y = layer.forward(ids, hid)
    assert y.shape == (0, 5, w.hc_mult, w.hidden)


def test_forward_flags_out_of_range_ids():
    w = W.small_workload(B=1, T=16)
    p = device_params(w)
    p.ids[0, 3] = w.vocab + 10
    layer = EngramLayer.from_params(p)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    layer.forward(p.ids, p.hidden, dev_status=st)
    assert L.engram_read_status(st) & L.STATUS_ID_RANGE


def test_forward_timeout_path_returns_and_context_survives():
    w = W.small_workload(B=2, T=64)
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    if not _tc_active(w):
        pytest.skip("tensor-core engine not active for this shape")
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.engram_set_debug(L.DEBUG_FORCE_TIMEOUT)
    try:
        layer.forward(p.ids, p.hidden, dev_status=st)
        bits = L.engram_read_status(st)
    finally:
        L.engram_set_debug(0)
    assert bits & L.STATUS_TIMEOUT
    # the context is still usable and the next call is correct
    y = _run(p)
    ref = oracle_forward_full(p)
    assert rel_err(y.double().cpu().numpy(), ref["Y"]) <= TOL["bf16"]


def _tc_active(w) -> bool:
    cfg = L.make_config(w.orders, w.heads_per_order, w.row_dim, w.hidden, w.hc_mult,
                        w.conv_kernel, w.dil, w.pad_id, w.vocab, w.torch_dtype)
    return L.engram_projection_engine(cfg) == L.ENGINE_TCGEN05
