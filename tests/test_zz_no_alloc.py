"""engram_forward_no_alloc: the whole pass in the library's static device
scratch, for callers that cannot allocate device memory (a plugin given only
its input and output buffers, or a latency-critical loop where cudaMalloc
would synchronise the device).

It must give what engram_forward gives with a caller workspace, on two calls
in a row (the shared scratch keeps the first call's contents), and reject a
batch whose scratch need exceeds the static array without launching.
Collected last on purpose; it needs nothing from the other tests.
"""
import pytest
import torch

from hashed_gram_conditional_hash_b200 import EngramLayer
from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W

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
    for y, ref in ((y1, ref1), (y2, ref2)):
        err = (y.double() - ref.double()).abs().max().item()
        assert err <= TOL_BF16 * ref.double().abs().max().item()


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
