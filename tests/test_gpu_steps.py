"""GPU parity of the single-step entry points against the oracle:
engram_compress_ids, engram_hash and engram_gather bit-exact;
engram_gate_fuse and engram_short_conv within the dtype tolerance."""
import numpy as np
import pytest
import torch

from hashed_gram_conditional_hash_b200 import _lib as L
from hashed_gram_conditional_hash_b200 import workloads as W
from oracle import engram_oracle as O

from gpu_helpers import TOL, device_params, oracle_ids, rel_err

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _cfg(w: W.Workload):
    return L.make_config(w.orders, w.heads_per_order, w.row_dim, w.hidden, w.hc_mult,
                         w.conv_kernel, w.dil, w.pad_id, w.vocab, w.torch_dtype,
                         w.rms_eps, w.gate_eps)


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def test_compress_bit_exact():
    w = W.CONFIGS["tiny_f32"]
    lut = torch.from_numpy(W.compress_lookup(w)).to(DEV)
    raw = torch.from_numpy(W.token_ids(w)).to(DEV)
    out = torch.empty_like(raw)
    st = _status()
    L.engram_compress_ids(raw, lut, out, st)
    assert L.engram_read_status(st) == 0
    np.testing.assert_array_equal(out.cpu().numpy(), O.compress_ids(raw.cpu().numpy(), lut.cpu().numpy()))
    bad = raw.clone()
    bad[0, 5] = 2048
    L.engram_compress_ids(bad, lut, out, st)
    assert L.engram_read_status(st) & L.STATUS_ID_RANGE
    assert int(out[0, 5]) == -1


@pytest.mark.parametrize("name", list(W.CONFIGS))
def test_hash_bit_exact_all_configs(name):
    w = W.CONFIGS[name]
    x = W.token_ids(w)
    if w.raw_vocab is not None:
        x = O.compress_ids(x, W.compress_lookup(w))
    primes, mult = W.head_primes(w), W.multipliers(w)
    ids = torch.from_numpy(x).to(DEV)
    idx = torch.empty((x.shape[0], x.shape[1], w.nh), dtype=torch.int64, device=DEV)
    st = _status()
    L.engram_hash(_cfg(w), ids, mult, primes, idx, dev_status=st)
    assert L.engram_read_status(st) == 0
    ref = O.ngram_hash(x, w.orders, w.heads_per_order, mult, primes, w.pad_id)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref)
    got = idx.cpu().numpy()
    assert np.all(got >= 0) and np.all(got < primes[None, None, :])


@pytest.mark.parametrize("B,T", [(1, 1), (2, 5), (3, 33), (2, 300), (5, 257)])
def test_hash_ragged_and_history(B, T):
    w = W.small_workload(orders=(2, 3, 4), heads_per_order=3)
    rng = np.random.default_rng(B * 1000 + T)
    x = rng.integers(0, w.vocab, size=(B, T))
    hist = rng.integers(0, w.vocab, size=(B, 3))
    primes, mult = W.head_primes(w), W.multipliers(w)
    idx = torch.empty((B, T, w.nh), dtype=torch.int64, device=DEV)
    for h in (None, hist):
        L.engram_hash(_cfg(w), torch.from_numpy(x).to(DEV), mult, primes, idx,
                      history=None if h is None else torch.from_numpy(h).to(DEV))
        ref = O.ngram_hash(x, w.orders, w.heads_per_order, mult, primes, w.pad_id, hist=h)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref)


def test_hash_flags_out_of_range_ids():
    w = W.small_workload()
    x = np.array([[1, 2, w.vocab, 4, -3, 6]])
    primes, mult = W.head_primes(w), W.multipliers(w)
    idx = torch.empty((1, 6, w.nh), dtype=torch.int64, device=DEV)
    st = _status()
    L.engram_hash(_cfg(w), torch.from_numpy(x).to(DEV), mult, primes, idx, dev_status=st)
    assert L.engram_read_status(st) & L.STATUS_ID_RANGE
    # bad ids hash as pad_id
    xf = x.copy()
    xf[0, 2] = w.pad_id
    xf[0, 4] = w.pad_id
    np.testing.assert_array_equal(idx.cpu().numpy(),
                                  O.ngram_hash(xf, w.orders, w.heads_per_order, mult, primes, w.pad_id))


@pytest.mark.parametrize("name", ["tiny_f32", "model_bf16", "large_table_bf16"])
def test_gather_bit_exact(name):
    w = W.CONFIGS[name]
    p = device_params(w)
    x = oracle_ids(p)
    idx_np = O.ngram_hash(x, w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
    M = x.size
    if M > 8192:  # large tables: a contiguous slab of tokens (all heads)
        idx_np = idx_np.reshape(M, -1)[:8192].reshape(1, 8192, -1)
        M = 8192
    idx = torch.from_numpy(idx_np).to(DEV)
    e = torch.empty((M, w.E), dtype=w.torch_dtype, device=DEV)
    st = _status()
    L.engram_gather(_cfg(w), p.table, p.offsets, idx, e, st)
    assert L.engram_read_status(st) == 0
    rows = (p.offsets[None, :] + idx_np.reshape(M, -1)).reshape(-1)
    fetched = p.table[torch.from_numpy(rows).to(DEV)].cpu()
    tab, _ = O.storage(fetched)
    ref = O.gather(tab, np.arange(w.nh) * 0, np.arange(M * w.nh).reshape(M, w.nh))
    got, _ = O.storage(e)
    np.testing.assert_array_equal(got, ref)


def test_gather_flags_bad_rows():
    w = W.small_workload()
    p = device_params(w)
    idx = torch.zeros((2, w.nh), dtype=torch.int64, device=DEV)
    idx[1, 0] = p.table.shape[0] + 5
    e = torch.full((2, w.E), 7.0, dtype=w.torch_dtype, device=DEV)
    st = _status()
    L.engram_gather(_cfg(w), p.table, p.offsets, idx, e, st)
    assert L.engram_read_status(st) & L.STATUS_ROW_RANGE
    assert torch.all(e[1, : w.row_dim] == 0)


@pytest.mark.parametrize("dtype,H,hc,M", [("bf16", 256, 2, 200), ("f32", 128, 3, 77),
                                          ("bf16", 512, 4, 1000)])
def test_gate_fuse_parity(dtype, H, hc, M):
    w = W.small_workload(dtype=dtype, hidden=H, hc_mult=hc)
    p = device_params(w)
    g = torch.Generator(device="cpu").manual_seed(3)
    e = (0.02 * torch.randn(M, w.E, generator=g)).to(w.torch_dtype).to(DEV)
    hid = torch.randn(M, hc, H, generator=g).to(w.torch_dtype).to(DEV)
    u = torch.empty((M, hc, H), dtype=w.torch_dtype, device=DEV)
    gates = torch.empty((M, hc), dtype=torch.float32, device=DEV)
    L.engram_gate_fuse(_cfg(w), e, p.w_value, p.w_key, p.norm_key, p.norm_query, hid, u, gates)
    torch.cuda.synchronize()
    V, s, gref = O.tokens_gate(O.widen(*O.storage(e)), H, hc, p.w_value.cpu(), p.w_key.cpu(),
                               p.norm_key.cpu(), p.norm_query.cpu(), hid.cpu(), w.rms_eps, w.gate_eps)
    uref = gref[:, :, None] * V[:, None, :]
    assert rel_err(u.double().cpu().numpy(), uref) <= TOL[dtype]
    mask = np.abs(s) >= 1e-5
    assert np.max(np.abs(gates.double().cpu().numpy() - gref)[mask]) <= TOL[dtype]


@pytest.mark.parametrize("engine", ["auto", "simt"])
def test_gate_is_one_half_exactly_when_a_branch_sees_zero_hidden(engine):
    # formulas page §2.2 step 2 with sign(0) = 0: a zero query gives s = 0,
    # hence g = sigmoid(0) = 1/2 exactly, and u = V/2 for that branch
    w = W.small_workload(hidden=512, hc_mult=4)
    p = device_params(w)
    M = 300
    g = torch.Generator(device="cpu").manual_seed(13)
    e = (0.02 * torch.randn(M, w.E, generator=g)).to(w.torch_dtype).to(DEV)
    hid = torch.randn(M, w.hc_mult, w.hidden, generator=g).to(w.torch_dtype)
    hid[:, 1] = 0
    hid = hid.to(DEV)
    u = torch.empty((M, w.hc_mult, w.hidden), dtype=w.torch_dtype, device=DEV)
    gates = torch.empty((M, w.hc_mult), dtype=torch.float32, device=DEV)
    L.engram_set_debug(L.DEBUG_FORCE_SIMT if engine == "simt" else 0)
    try:
        L.engram_gate_fuse(_cfg(w), e, p.w_value, p.w_key, p.norm_key, p.norm_query, hid, u, gates)
        torch.cuda.synchronize()
    finally:
        L.engram_set_debug(0)
    assert torch.all(gates[:, 1] == 0.5)
    V, s, gref = O.tokens_gate(O.widen(*O.storage(e)), w.hidden, w.hc_mult, p.w_value.cpu(), p.w_key.cpu(),
                               p.norm_key.cpu(), p.norm_query.cpu(), hid.cpu(), w.rms_eps, w.gate_eps)
    assert np.all(s[:, 1] == 0.0) and np.all(gref[:, 1] == 0.5)
    assert rel_err(u.double().cpu().numpy(), gref[:, :, None] * V[:, None, :]) <= TOL["bf16"]
    # the other branches keep their gates (masking the sign-ambiguous |s| < 1e-5)
    mask = np.abs(s) >= 1e-5
    assert np.max(np.abs(gates.double().cpu().numpy() - gref)[mask]) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_short_conv_parity_and_state(dtype):
    w = W.small_workload(dtype=dtype, hidden=128, hc_mult=2)
    p = device_params(w)
    B, T, Cc = 3, 40, w.hc_mult * w.hidden
    g = torch.Generator(device="cpu").manual_seed(5)
    u = torch.randn(B, T, Cc, generator=g).to(w.torch_dtype).to(DEV)
    y = torch.empty_like(u)
    cfg = _cfg(w)
    L.engram_short_conv(cfg, u, p.conv_w, y)
    torch.cuda.synchronize()
    ud = u.double().cpu().numpy()
    ref = O.short_conv(ud, p.conv_w.double().cpu().numpy(), w.conv_kernel, w.dil)
    assert rel_err(y.double().cpu().numpy(), ref) <= TOL[dtype]
    # chunked with a state: [0, 17) then [17, 40) equals the whole
    R = (w.conv_kernel - 1) * w.dil
    state = torch.zeros((B, R, Cc), dtype=w.torch_dtype, device=DEV)
    y1 = torch.empty((B, 17, Cc), dtype=w.torch_dtype, device=DEV)
    y2 = torch.empty((B, 23, Cc), dtype=w.torch_dtype, device=DEV)
    L.engram_short_conv(cfg, u[:, :17].contiguous(), p.conv_w, y1, conv_state=state)
    L.engram_short_conv(cfg, u[:, 17:].contiguous(), p.conv_w, y2, conv_state=state)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat([y1, y2], 1), y)
    assert torch.equal(state, u[:, T - R:])
