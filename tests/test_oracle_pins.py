"""Pins of the float64 oracle to facts the pages and the mathematics fix.

Each test ties one oracle step to something other than the oracle itself: the
worked example printed on the formulas page (§4.3), closed forms, special
cases that reduce to integer arithmetic, a textbook routine or a library
routine (numpy take / matmul, torch rms_norm / conv1d), invariants, and
brute force on tiny inputs.  The cases are chosen so that a plausible slip in
the oracle (a dropped term, a swapped index or operand, a wrong sign, add
instead of xor, sqrt(E) instead of sqrt(H), eps added instead of floored) fails
at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import engram_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")
BIGP = 1_000_003  # a prime above every mix value used in the exact-value pins


def _read_fixture(name):
    out = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            out[k] = [int(x) for x in v]
    return out


# ---------------------------------------------------------------- a2 shift

def test_shift_worked_example():
    fx = _read_fixture("shift_pad_example.txt")
    x = np.array([fx["sequence"]], dtype=np.int64)
    pad = fx["pad"][0]
    for k in range(3):
        np.testing.assert_array_equal(O.shift(x, k, pad)[0], fx["shift%d" % k])
    # the 3-gram at position 2, read oldest first from shift_2, shift_1, shift_0
    gram = [int(O.shift(x, k, pad)[0, 2]) for k in (2, 1, 0)]
    assert gram == fx["ngram_at_2"]


def test_shift_history_continues_sequence():
    rng = np.random.default_rng(0)
    full = rng.integers(0, 50, size=(2, 12))
    hist, tail = full[:, 5:8], full[:, 8:]
    for k in range(4):
        np.testing.assert_array_equal(O.shift(tail, k, pad_id=-5, hist=hist),
                                      O.shift(full, k, pad_id=-5)[:, 8:])


# ---------------------------------------------------------------- a3 hash

def test_hash_position0_is_modular_product():
    # At t = 0 every earlier token is the pad id; with pad = 0 the xor mix
    # collapses to t_0 * m_0 (the current token takes m_0).
    x = np.array([[123457, 9, 9, 9]])
    mult = [2 ** 31 - 1, 3, 5]
    primes = [1_000_003, 65_537, 97]
    idx = O.ngram_hash(x, orders=(3,), J=3, mult=mult, primes=primes, pad_id=0)
    for j, p in enumerate(primes):
        assert idx[0, 0, j] == (123457 * (2 ** 31 - 1)) % p


def test_hash_token_to_multiplier_assignment():
    # Multipliers with disjoint bit ranges make xor equal to a sum, so the
    # index reveals which token met which multiplier: t_k = x[t-k] meets m_k.
    x = np.array([[11, 22, 33, 44]])
    mult = [1, 1 << 20, 1 << 40]
    p = (1 << 61) - 1  # prime above every mix here
    idx = O.ngram_hash(x, orders=(2, 3), J=1, mult=mult, primes=[p, p], pad_id=0)
    assert idx[0, 1, 0] == 22 + (11 << 20)                       # bigram at t=1
    assert idx[0, 2, 1] == 33 + (22 << 20) + (11 << 40)          # trigram at t=2
    assert idx[0, 3, 1] == 44 + (33 << 20) + (22 << 40)          # trigram at t=3
    assert idx[0, 1, 1] == 22 + (11 << 20) + (0 << 40)           # pad enters at t=1


def test_hash_mixes_with_xor_not_add():
    x = np.array([[5, 3, 6]])
    idx = O.ngram_hash(x, orders=(2, 3), J=1, mult=[1, 1, 1], primes=[BIGP, BIGP], pad_id=0)
    assert idx[0, 1, 0] == (3 ^ 5)          # 6, an add would give 8
    assert idx[0, 2, 1] == (6 ^ 3 ^ 5)      # 0


def test_hash_heads_differ_only_by_prime():
    rng = np.random.default_rng(3)
    x = rng.integers(0, 1000, size=(2, 40))
    p1 = [10007, 10009, 10037]
    big = (1 << 61) - 1
    mult = [7, 9, 11]
    idx = O.ngram_hash(x, orders=(3,), J=3, mult=mult, primes=p1, pad_id=0)
    mix = O.ngram_hash(x, orders=(3,), J=1, mult=mult, primes=[big], pad_id=0)[..., 0]
    for j, p in enumerate(p1):
        np.testing.assert_array_equal(idx[..., j], mix % p)


def test_hash_range_and_brute_force_dict():
    # Tiny vocab: many positions share an n-gram; the index must be a function
    # of the n-gram tuple alone, and lie in [0, p).
    rng = np.random.default_rng(1)
    x = rng.integers(0, 5, size=(3, 64))
    orders, J = (2, 3), 3
    primes = [101, 103, 107, 109, 113, 127]
    mult = [2 * int(r) + 1 for r in rng.integers(0, 1 << 30, size=3)]
    pad = 2
    idx = O.ngram_hash(x, orders, J, mult, primes, pad)
    seen = {}
    for b in range(3):
        for t in range(64):
            for o, n in enumerate(orders):
                gram = tuple(int(x[b, t - k]) if t - k >= 0 else pad for k in range(n))
                for j in range(J):
                    h = o * J + j
                    v = int(idx[b, t, h])
                    assert 0 <= v < primes[h]
                    key = (h, gram)
                    assert seen.setdefault(key, v) == v
    # and with small multipliers each value is the xor/mod computed by hand
    # on Python integers for a handful of grams
    for (h, gram), v in list(seen.items())[:40]:
        o = h // J
        mix = 0
        for k, tk in enumerate(gram):
            mix ^= tk * mult[k]
        assert v == mix % primes[h]


def test_hash_matches_numpy_int64_semantics():
    # The pages' snippets run on NumPy int64; large multipliers wrap there.
    rng = np.random.default_rng(5)
    x = rng.integers(0, 1 << 40, size=(2, 30))
    mult = rng.integers(1 << 40, 1 << 62, size=4)
    primes = [1_000_003, 999_983, (1 << 31) - 1, 4_194_319]
    idx = O.ngram_hash(x, orders=(2, 4), J=2, mult=mult, primes=primes, pad_id=17)
    with np.errstate(over="ignore"):
        for o, n in enumerate((2, 4)):
            toks = [np.pad(x, ((0, 0), (k, 0)), constant_values=17)[:, :30] for k in range(n)]
            mix = toks[0] * mult[0]
            for k in range(1, n):
                mix = np.bitwise_xor(mix, toks[k] * mult[k])
            for j in range(2):
                np.testing.assert_array_equal(idx[..., o * 2 + j], np.mod(mix, primes[o * 2 + j]))


def test_hash_with_history_equals_longer_prefill():
    rng = np.random.default_rng(9)
    x = rng.integers(0, 300, size=(4, 20))
    kw = dict(orders=(2, 3, 4), J=2, mult=[3, 5, 7, 9], primes=[31, 37, 41, 43, 47, 53], pad_id=1)
    full = O.ngram_hash(x, **kw)
    part = O.ngram_hash(x[:, 12:], hist=x[:, 9:12], **kw)
    np.testing.assert_array_equal(part, full[:, 12:])


# ---------------------------------------------------------------- a1, a4

def test_compress_and_gather_match_numpy_take():
    rng = np.random.default_rng(2)
    lut = rng.integers(0, 50, size=80)
    raw = rng.integers(0, 80, size=(2, 9))
    np.testing.assert_array_equal(O.compress_ids(raw, lut), np.take(lut, raw))
    table = rng.integers(0, 1 << 16, size=(40, 8)).astype(np.uint16)
    offs = np.array([0, 11, 24])
    idx = np.stack([rng.integers(0, 11, 10), rng.integers(0, 13, 10), rng.integers(0, 16, 10)], -1)
    e = O.gather(table, offs, idx)
    ref = table[offs[None, :] + idx].reshape(10, -1)
    np.testing.assert_array_equal(e, ref)
    assert e.dtype == np.uint16


# ---------------------------------------------------------------- sharded table

def test_shard_route_hand_example():
    # rows 5 2 7 4 0 3 over 3 shards: owners 2 2 1 1 0 0, local rows 1 0 2 1 0 1
    counts, req_rows, req_pos = O.shard_route(np.array([5, 2, 7, 4, 0, 3]), 3)
    assert counts.tolist() == [2, 2, 2]
    assert req_pos.tolist() == [4, 5, 2, 3, 0, 1]
    assert req_rows.tolist() == [0, 1, 2, 1, 1, 0]


def test_shard_route_brute_force_and_reassembly():
    rng = np.random.default_rng(5)
    table = rng.integers(0, 1 << 16, size=(97, 8)).astype(np.uint16)
    rows = rng.integers(0, 97, size=300)
    for R in (1, 2, 3, 8):
        counts, req_rows, req_pos = O.shard_route(rows, R)
        # brute force: walk q in order, append to its shard's list
        lists = [[] for _ in range(R)]
        for q, row in enumerate(rows.tolist()):
            lists[row % R].append((row // R, q))
        flat = [x for lst in lists for x in lst]
        assert counts.tolist() == [len(l) for l in lists]
        assert req_rows.tolist() == [a for a, _ in flat]
        assert req_pos.tolist() == [b for _, b in flat]
        # serving each shard's requests from its shard and placing them at
        # req_pos gives the plain gather of the full table
        shards = [O.shard_table(table, R, r) for r in range(R)]
        assert sum(len(sh) for sh in shards) == len(table)
        owner = np.repeat(np.arange(R), counts)
        got = np.stack([shards[o][k] for o, k in zip(owner, req_rows)])
        e = np.empty_like(table[rows])
        e[req_pos] = got
        np.testing.assert_array_equal(e, table[rows])
    c1, r1, p1 = O.shard_route(rows, 1)
    np.testing.assert_array_equal(r1, rows)
    np.testing.assert_array_equal(p1, np.arange(len(rows)))


def test_widen_bf16_is_exact():
    t = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    a, code = O.storage(t)
    np.testing.assert_array_equal(O.widen(a, code), t.double().numpy())


# ---------------------------------------------------------------- a5-a7

def _gate_inputs(n=5, E=48, H=64, hc=3, seed=0, dtype=torch.float32, norm_std=0.1):
    g = torch.Generator().manual_seed(seed)
    e = torch.randn(n, E, generator=g, dtype=torch.float64)
    wv = torch.randn(H, E, generator=g).to(dtype)
    wk = torch.randn(hc, H, E, generator=g).to(dtype)
    nk = (1 + norm_std * torch.randn(hc, H, generator=g)).to(dtype)
    nq = (1 + norm_std * torch.randn(hc, H, generator=g)).to(dtype)
    hid = torch.randn(n, hc, H, generator=g).to(dtype)
    return e, wv, wk, nk, nq, hid


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_projection_matches_numpy_matmul(dtype):
    e, wv, wk, nk, nq, hid = _gate_inputs(dtype=dtype)
    V, s, g = O.tokens_gate(e.numpy(), 64, 3, wv, wk, nk, nq, hid, 1e-6, 1e-6)
    np.testing.assert_allclose(V, e.numpy() @ wv.double().numpy().T, rtol=1e-12, atol=1e-12)


def test_projection_one_hot_selects_column():
    e, wv, wk, nk, nq, hid = _gate_inputs()
    oh = np.zeros((1, 48))
    oh[0, 17] = 1.0
    V, _, _ = O.tokens_gate(oh, 64, 3, wv, wk, nk, nq, hid[:1], 1e-6, 1e-6)
    np.testing.assert_array_equal(V[0], wv[:, 17].double().numpy())


def test_rmsnorm_matches_torch():
    x = np.random.default_rng(4).normal(size=96)
    w = np.random.default_rng(5).normal(1, 0.1, size=96)
    ref = F.rms_norm(torch.from_numpy(x), (96,), torch.from_numpy(w), eps=1e-6).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, w, 1e-6), ref, rtol=1e-13)


def test_score_closed_form_parallel_and_antiparallel():
    # K_h parallel to Q_h with unit norm weights and eps = 0 gives
    # s = sqrt(H) * cos = sqrt(H) (pins the divisor: H = 64, E = 48).
    e, wv, wk, nk, nq, hid = _gate_inputs(n=1, norm_std=0.0)
    K = (wk.double() @ e[0]).float()                        # [hc, H]
    for scale, want in ((2.5, math.sqrt(64)), (-0.75, -math.sqrt(64))):
        hid1 = (scale * K).unsqueeze(0).float()
        # K was rounded to fp32 for the hidden state; that leaves cos = 1 - O(1e-14)
        _, s, g = O.tokens_gate(e[:1].numpy(), 64, 3, wv, wk, torch.ones(3, 64),
                                torch.ones(3, 64), hid1, 0.0, 1e-6)
        np.testing.assert_allclose(s[0], want, rtol=1e-6)


def test_score_zero_query_gives_half_gate():
    e, wv, wk, nk, nq, hid = _gate_inputs(n=2)
    _, s, g = O.tokens_gate(e[:2].numpy(), 64, 3, wv, wk, nk, nq, torch.zeros(2, 3, 64), 1e-6, 1e-6)
    assert np.all(s == 0.0) and np.all(g == 0.5)


def test_score_norm_weights_enter_once_each():
    e, wv, wk, nk, nq, hid = _gate_inputs(n=3, norm_std=0.0)
    ones = torch.ones(3, 64)
    _, s1, _ = O.tokens_gate(e[:3].numpy(), 64, 3, wv, wk, ones, ones, hid[:3], 1e-6, 1e-6)
    _, s2, _ = O.tokens_gate(e[:3].numpy(), 64, 3, wv, wk, 2 * ones, 3 * ones, hid[:3], 1e-6, 1e-6)
    np.testing.assert_allclose(s2, 6 * s1, rtol=1e-12)
    # scale invariance of RMSNorm (eps = 0): scaling the hidden state leaves s
    _, s3, _ = O.tokens_gate(e[:3].numpy(), 64, 3, wv, wk, ones, ones, 8 * hid[:3], 0.0, 1e-6)
    _, s4, _ = O.tokens_gate(e[:3].numpy(), 64, 3, wv, wk, ones, ones, hid[:3], 0.0, 1e-6)
    np.testing.assert_allclose(s3, s4, rtol=1e-12)


def test_score_matches_torch_composition():
    e, wv, wk, nk, nq, hid = _gate_inputs(n=4)
    V, s, g = O.tokens_gate(e[:4].numpy(), 64, 3, wv, wk, nk, nq, hid[:4], 1e-6, 1e-6)
    K = torch.einsum("nE,cHE->ncH", e[:4], wk.double())
    Kn = F.rms_norm(K, (64,), None, eps=1e-6) * nk.double()
    Qn = F.rms_norm(hid[:4].double(), (64,), None, eps=1e-6) * nq.double()
    sref = (Kn * Qn).sum(-1) / math.sqrt(64)
    np.testing.assert_allclose(s, sref.numpy(), rtol=1e-10, atol=1e-12)


def test_gate_special_values():
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    assert O.gate_value(0.0) == 0.5
    assert O.gate_value(4.0) == pytest.approx(sig(2.0), rel=1e-15, abs=0)
    assert O.gate_value(2.25) == pytest.approx(sig(1.5), rel=1e-15, abs=0)
    # |s| below 1e-6 is floored (not shifted by eps): sqrt(1e-6) = 1e-3
    assert O.gate_value(1e-8) == pytest.approx(sig(1e-3), rel=1e-15, abs=0)
    assert O.gate_value(-1e-8) == pytest.approx(sig(-1e-3), rel=1e-15, abs=0)
    # above the floor the magnitude is untouched: sqrt(4 + 1e-6) would differ
    assert abs(O.gate_value(4.0) - sig(math.sqrt(4.0 + 1e-6))) > 1e-9
    for s in (1e-9, 0.3, 2.0, 17.0, 1e4):
        assert O.gate_value(-s) == pytest.approx(1.0 - O.gate_value(s), abs=1e-15)
    ss = np.linspace(-50, 50, 1001)
    gs = np.array([O.gate_value(v) for v in ss])
    assert np.all(np.diff(gs) >= 0) and np.all((gs > 0) & (gs < 1))


# ---------------------------------------------------------------- a8, a9

def _u(B=2, T=30, C=6, seed=0):
    return np.random.default_rng(seed).normal(size=(B, T, C))


def test_conv_zero_weights_is_identity():
    U = _u()
    np.testing.assert_array_equal(O.short_conv(U, np.zeros((6, 4)), 4, 3), U)


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_conv_one_hot_tap_is_residual_plus_shift(tap):
    U = _u()
    w = np.zeros((6, 4))
    w[:, tap] = 1.0
    d = (3 - tap) * 3
    sh = np.zeros_like(U)
    sh[:, d:] = U[:, : U.shape[1] - d]
    np.testing.assert_array_equal(O.short_conv(U, w, 4, 3), U + sh)


def test_conv_matches_torch_conv1d():
    U = _u(T=50, C=8)
    w = np.random.default_rng(1).normal(size=(8, 4))
    for dil in (1, 3, 4):
        x = torch.from_numpy(U).transpose(1, 2)
        ref = F.conv1d(x, torch.from_numpy(w)[:, None, :], padding=3 * dil, dilation=dil, groups=8)
        ref = ref[..., :50].transpose(1, 2).numpy() + U
        np.testing.assert_allclose(O.short_conv(U, w, 4, dil), ref, rtol=1e-12, atol=1e-12)


def test_conv_is_causal_and_state_continues():
    U = _u(T=40)
    w = np.random.default_rng(2).normal(size=(6, 4))
    Y = O.short_conv(U, w, 4, 3)
    U2 = U.copy()
    U2[:, 25] += 10.0
    Y2 = O.short_conv(U2, w, 4, 3)
    np.testing.assert_array_equal(Y[:, :25], Y2[:, :25])
    assert np.all(Y[:, 25] != Y2[:, 25])
    Yb = O.short_conv(U[:, 20:], w, 4, 3, prev=U[:, 11:20])
    np.testing.assert_allclose(Yb, Y[:, 20:], rtol=0, atol=0)


def test_conv_point_agrees_with_short_conv_of_gated_value():
    rng = np.random.default_rng(6)
    T, H, hc, K, dil = 20, 5, 3, 4, 3
    V = rng.normal(size=(T, H))
    g = rng.uniform(0.1, 0.9, size=(T, hc))
    w = rng.normal(size=(hc * H, K)).astype(np.float32)
    U = (g[:, :, None] * V[:, None, :]).reshape(1, T, hc * H)          # a8
    Y = O.short_conv(U, w.astype(np.float64), K, dil).reshape(T, hc, H)
    for t in (0, 4, 9, 19):
        taps = [t - (K - 1 - i) * dil for i in range(K)]
        valid = np.array([tp >= 0 for tp in taps], dtype=np.int32)
        Vt = np.array([V[tp] if tp >= 0 else np.zeros(H) for tp in taps])
        gt = np.array([g[tp] if tp >= 0 else np.zeros(hc) for tp in taps])
        np.testing.assert_allclose(O.conv_point(Vt, gt, valid, w), Y[t], rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- whole pass

def _tiny(**kw):
    from hashed_gram_conditional_hash_b200 import workloads as W
    w = W.small_workload(**kw)
    return w, W.make_params(w, "cpu")


def _run_forward(w, p, **over):
    x = p.ids.numpy()
    if p.lookup is not None:
        x = O.compress_ids(x, p.lookup.numpy())
    args = dict(x=x, orders=w.orders, J=w.heads_per_order, mult=p.mult, primes=p.primes,
                row_offsets=p.offsets, pad_id=w.pad_id, table=p.table, w_value=p.w_value,
                w_key=p.w_key, norm_key=p.norm_key, norm_query=p.norm_query, conv_w=p.conv_w,
                hidden=p.hidden, K=w.conv_kernel, dil=w.dil)
    args.update(over)
    return O.forward(**args)


def test_forward_composes_the_steps():
    w, p = _tiny(B=2, T=19, dtype="f32", row_dim=16, hidden=64)
    out = _run_forward(w, p)
    x = p.ids.numpy()
    idx = O.ngram_hash(x, w.orders, w.heads_per_order, p.mult, p.primes, w.pad_id)
    np.testing.assert_array_equal(out["idx"], idx)
    e = p.table.double().numpy()[p.offsets[None, None, :] + idx].reshape(2, 19, -1)
    np.testing.assert_allclose(out["V"], e @ p.w_value.double().numpy().T, rtol=1e-12, atol=1e-13)
    U = (out["g"][..., None] * out["V"][:, :, None, :]).reshape(2, 19, -1)
    Y = O.short_conv(U, p.conv_w.double().numpy(), 4, w.dil)
    np.testing.assert_allclose(out["Y"].reshape(2, 19, -1), Y, rtol=1e-12, atol=1e-13)


def test_forward_zero_conv_is_gated_value():
    w, p = _tiny(B=1, T=11)
    out = _run_forward(w, p, conv_w=torch.zeros_like(p.conv_w))
    np.testing.assert_array_equal(out["Y"], out["g"][..., None] * out["V"][:, :, None, :])


def test_forward_identical_branches_agree():
    w, p = _tiny(B=1, T=13, hc_mult=4, dtype="f32")
    hc = 4
    out = _run_forward(w, p, w_key=p.w_key[:1].repeat(hc, 1, 1), norm_key=p.norm_key[:1].repeat(hc, 1),
                       norm_query=p.norm_query[:1].repeat(hc, 1),
                       hidden=p.hidden[:, :, :1].repeat(1, 1, hc, 1),
                       conv_w=p.conv_w[: w.hidden].repeat(hc, 1))
    for h in range(1, hc):
        np.testing.assert_array_equal(out["Y"][:, :, h], out["Y"][:, :, 0])


def test_forward_sampled_agrees_with_forward():
    w, p = _tiny(B=2, T=23)
    out = _run_forward(w, p)
    pos = [(0, 0), (0, 5), (1, 9), (1, 22)]
    tab = p.table
    Y, s, g, idx = O.forward_sampled(
        p.ids.numpy(), pos, w.orders, w.heads_per_order, p.mult, p.primes, p.offsets,
        w.pad_id, fetch_rows=lambda r: tab[torch.from_numpy(r)],
        fetch_hidden=lambda b, t: p.hidden[torch.from_numpy(b), torch.from_numpy(t)],
        w_value=p.w_value, w_key=p.w_key, norm_key=p.norm_key, norm_query=p.norm_query,
        conv_w=p.conv_w, K=4, dil=w.dil)
    for n, (b, t) in enumerate(pos):
        np.testing.assert_allclose(Y[n], out["Y"][b, t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(g[n], out["g"][b, t], rtol=1e-13)
