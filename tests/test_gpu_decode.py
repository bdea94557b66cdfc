"""Streaming (decode) parity: the decode workload's 1024 sequences advance one
token per engram_forward call for 256 calls, carrying the id ring and the
V/gate rings in an engram_state.  Checked against the oracle's prefill over the
same 256-token sequences at sampled positions, and against this library's own
prefill over T = 256 (same kernels, so agreement is to rounding of identical
operations), plus chunked prefill with the state, whose concatenated output is
checked against the oracle's prefill over the whole sequence."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_hash_b200 import EngramLayer
from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W

from gpu_helpers import TOL, device_params, oracle_at, oracle_forward_full, rel_err, sample_positions

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_all(layer, ids_bt, hidden_tb):
    """ids_bt [B, S] (device), hidden_tb [S, B, hc, H] -> Y [S, B, hc, H]."""
    B, S = ids_bt.shape
    state = layer.new_state(B)
    ws = layer.workspace(B, 1)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    steps = ids_bt.t().contiguous().view(S, B, 1)
    ys = torch.empty((S, B, 1, layer.hc, layer.hidden), dtype=layer.dtype, device=DEV)
    for c in range(S):
        # each step's ids in a buffer of their own: the ABI takes 16-byte aligned
        # pointers, and a row of the [S, B] view starts at c * B * 8 bytes
        layer.forward(steps[c].clone(), hidden_tb[c].view(B, 1, layer.hc, layer.hidden), y=ys[c],
                      ws=ws, state=state, dev_status=st)
    assert L.engram_read_status(st) == 0
    assert torch.all(state.pos == S)
    return ys.view(S, B, layer.hc, layer.hidden), state


def test_decode_workload_matches_oracle_and_prefill():
    w = W.CONFIGS["decode_bf16"]
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    ys, state = _decode_all(layer, p.ids, p.hidden)
    S, B = w.decode_calls, w.B
    # oracle: the prefill over the 256-token sequences at sampled positions
    pos = sample_positions(B, S, w.dil, 4096, seed=5)
    Yref, _, _, _ = oracle_at(p, pos, hidden_bt=lambda b, t: p.hidden[torch.from_numpy(t).to(DEV),
                                                                         torch.from_numpy(b).to(DEV)])
    got = torch.stack([ys[t, b] for b, t in pos]).double().cpu().numpy()
    assert rel_err(got, Yref) <= TOL["bf16"]
    # this library's prefill over T = 256 for a slice of the sequences
    nb = 64
    y_pre = layer.forward(p.ids[:nb].contiguous(), p.hidden[:, :nb].transpose(0, 1).contiguous())
    y_dec = ys[:, :nb].transpose(0, 1)
    err = (y_pre.double() - y_dec.double()).abs().max().item()
    assert err <= 1e-2 * y_pre.double().abs().max().item()
    # the id ring holds the last max_n - 1 ids of every sequence
    assert torch.equal(state.id_ring, p.ids[:, S - (w.max_n - 1):])


@pytest.mark.parametrize("chunks", [(5, 1, 13, 2, 40), (64,), (1,) * 9 + (55,), (10, 70, 64)])
def test_chunked_prefill_with_state(chunks):
    w = W.small_workload(B=3, T=sum(chunks), orders=(2, 3, 4), dilation=4, hidden=256, hc_mult=2)
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    y_full = layer.forward(p.ids, p.hidden)
    state = layer.new_state(w.B)
    outs, t0 = [], 0
    for n in chunks:
        ids = p.ids[:, t0:t0 + n].contiguous()
        hid = p.hidden[:, t0:t0 + n].contiguous()
        outs.append(layer.forward(ids, hid, state=state))
        t0 += n
    y = torch.cat(outs, 1)
    err = (y.double() - y_full.double()).abs().max().item()
    assert err <= 1e-2 * y_full.double().abs().max().item()
    assert torch.all(state.pos == t0)
    # the chunks together are the oracle's prefill over the whole sequence
    ref = oracle_forward_full(p)
    assert rel_err(y.double().cpu().numpy(), ref["Y"]) <= TOL[w.dtype]


@pytest.mark.parametrize("B,hc,hidden,dil,orders", [(9, 1, 512, 3, (2, 3)), (17, 4, 768, 2, (2,)),
                                                     (8, 3, 256, 5, (2, 3, 5)), (5, 2, 256, 8, (1, 8))])
def test_decode_steps_partial_blocks_and_branch_counts(B, hc, hidden, dil, orders):
    # every token a decode step (T = 1 with the state): batches that leave the
    # decode conv's last block of sequences partly empty, one to four branches,
    # several 256-channel slices, dilations whose ring wraps several times
    T = 40
    w = W.small_workload(B=B, T=T, orders=orders, dilation=dil, hidden=hidden, hc_mult=hc)
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    ys, state = _decode_all(layer, p.ids, p.hidden.transpose(0, 1).contiguous())
    y = ys.transpose(0, 1)                                  # [B, T, hc, H]
    y_pre = layer.forward(p.ids, p.hidden)
    err = (y.double() - y_pre.double()).abs().max().item()
    assert err <= 1e-2 * y_pre.double().abs().max().item()
    assert rel_err(y.double().cpu().numpy(), oracle_forward_full(p)["Y"]) <= TOL[w.dtype]
    assert torch.all(state.pos == T)


def test_streaming_with_raw_ids_keeps_compressed_ids_in_the_ring():
    # raw ids go through the lookup; the ring keeps the compressed ids the
    # hash needs for the next chunk (decode steps, then one long chunk)
    w = W.small_workload(B=3, T=80, raw_vocab=6500, orders=(2, 3, 4), dilation=4, hidden=256, hc_mult=2)
    p = device_params(w)
    layer = EngramLayer.from_params(p)
    y_full = layer.forward(p.ids, p.hidden)
    state = layer.new_state(w.B)
    outs, t0 = [], 0
    for n in (1,) * 5 + (75,):
        outs.append(layer.forward(p.ids[:, t0:t0 + n].contiguous(), p.hidden[:, t0:t0 + n].contiguous(),
                                  state=state))
        t0 += n
    y = torch.cat(outs, 1)
    err = (y.double() - y_full.double()).abs().max().item()
    assert err <= 1e-2 * y_full.double().abs().max().item()
    assert rel_err(y.double().cpu().numpy(), oracle_forward_full(p)["Y"]) <= TOL[w.dtype]
    assert torch.equal(state.id_ring, p.lookup[p.ids[:, -(w.max_n - 1):]])
    assert torch.all(state.pos == w.T)
