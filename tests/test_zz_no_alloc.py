"""engram_forward_no_alloc: the whole pass in the library's static device
scratch, for callers that cannot allocate device memory (a plugin given only
its input and output buffers, or a latency-critical loop where cudaMalloc
would synchronise the device).

It must give what engram_forward gives with a caller workspace, on two calls
in a row (the shared scratch keeps the first call's contents), and what the
float64 oracle gives; the streaming state (decode steps, whose scratch need
sets the array's size) and the fused-gather workspace layout must work in it
too; a batch whose scratch need exceeds the static array is rejected without
launching.  Collected last on purpose; it needs nothing from the other tests.
"""
import pytest
import torch

from hashed_gram_conditional_hash_b200 import EngramLayer
from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W

from gpu_helpers import oracle_forward_full, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"
TOL_BF16 = 2e-2


def _both(layer, ids, hidden):
    ref = layer.forward(ids, hidden)
    y = torch.full_like(ref, float("nan"))
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    L.engram_forward_no_alloc(layer.cfg, layer.weights, ids, hidden, y, dev_status=st)
    assert L.engram_read_status(st) == 0
    return y, ref


def test_no_alloc_matches_forward_on_two_calls():
    w1 = W.small_workload(B=3, T=150, hidden=512, hc_mult=4)
    p1 = W.make_params(w1, DEV)
    layer1 = EngramLayer.from_params(p1)
    assert L.engram_forward_workspace_size(layer1.cfg, w1.B, w1.T) <= L.NO_ALLOC_SCRATCH_BYTES
    y1, ref1 = _both(layer1, p1.ids, p1.hidden)
    # second call: another layer and batch shape, reusing the same scratch
    w2 = W.small_workload(B=2, T=97, hidden=256, hc_mult=2, orders=(2, 3, 4), dilation=4, seed=9)
    p2 = W.make_params(w2, DEV)
    layer2 = EngramLayer.from_params(p2)
    y2, ref2 = _both(layer2, p2.ids, p2.hidden)
    for y, ref, p in ((y1, ref1, p1), (y2, ref2, p2)):
        err = (y.double() - ref.double()).abs().max().item()
        assert err <= TOL_BF16 * ref.double().abs().max().item()
        assert rel_err(y.double().cpu().numpy(), oracle_forward_full(p)["Y"]) <= TOL_BF16


def test_no_alloc_decode_steps_match_forward():
    # one decode step of 256 sequences, twice in a row, through the static
    # array and through a caller workspace, each with its own copy of the state
    w = W.small_workload(B=256, T=2, hidden=512, hc_mult=4, orders=(2, 3, 4), dilation=4)
    p = W.make_params(w, DEV)
    layer = EngramLayer.from_params(p)
    s_ref, s_na = layer.new_state(w.B), layer.new_state(w.B)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    for t in range(w.T):
        ids = p.ids[:, t:t + 1].contiguous()
        hid = p.hidden[:, t:t + 1].contiguous()
        ref = layer.forward(ids, hid, state=s_ref)
        y = torch.full_like(ref, float("nan"))
        L.engram_forward_no_alloc(layer.cfg, layer.weights, ids, hid, y, state=s_na.c, dev_status=st)
        assert L.engram_read_status(st) == 0
        assert torch.equal(y, ref)
    for a, b in ((s_na.id_ring, s_ref.id_ring), (s_na.v_ring, s_ref.v_ring), (s_na.g_ring, s_ref.g_ring),
                 (s_na.pos, s_ref.pos)):
        assert torch.equal(a, b)


def test_no_alloc_fused_gather_layout():
    # the fused-gather path keeps head-major table rows where e would be
    w = W.small_workload(B=2, T=130, hidden=512, hc_mult=4)
    p = W.make_params(w, DEV)
    layer = EngramLayer.from_params(p)
    L.engram_set_debug(L.DEBUG_FUSED_GATHER)
    try:
        y, ref = _both(layer, p.ids, p.hidden)
    finally:
        L.engram_set_debug(0)
    assert torch.equal(y, ref)
    assert rel_err(y.double().cpu().numpy(), oracle_forward_full(p)["Y"]) <= TOL_BF16


def test_no_alloc_rejects_batch_beyond_static_scratch():
    w = W.small_workload(B=64, T=2048, hidden=1024, hc_mult=4)
    cfg = L.make_config(w.orders, w.heads_per_order, w.row_dim, w.hidden, w.hc_mult,
                        w.conv_kernel, w.dil, w.pad_id, w.vocab, w.torch_dtype)
    assert L.engram_forward_workspace_size(cfg, w.B, w.T) > L.NO_ALLOC_SCRATCH_BYTES
    weights = L.EngramWeights()
    before = L.engram_launch_count()
    with pytest.raises(L.EngramError) as ei:
        L.engram_forward_no_alloc(cfg, weights, torch.zeros((w.B, w.T), dtype=torch.int64, device=DEV),
                                  torch.empty(0, device=DEV), torch.empty(0, device=DEV))
    assert ei.value.code == 1 and "split the batch" in str(ei.value)
    assert L.engram_launch_count() == before
