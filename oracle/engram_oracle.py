"""NumPy driver for the float64 C oracle of the Engram forward pass.

TEST INFRASTRUCTURE ONLY: imported by tests/, ``__graft_entry__.smoke()`` and
the CPU-baseline / reference legs of ``bench.py``.  It shares nothing with the
CUDA library (no code, no constants, no helpers) and never calls it.

The C file ``engram_oracle.c`` holds every step of the method (see its header
for the page and section each function follows).  This module only marshals
arrays and composes the C steps:

* ``forward``          - the whole pass over [B, T] with every input on the host;
* ``forward_sampled``  - Y at chosen (b, t) positions only, for workloads whose
                         tables live on a device: the caller supplies a row
                         fetcher, the oracle does the arithmetic;
* ``shard_table``, ``shard_route`` - the table split over R devices and the
                         requests each device sends to the others (plain numpy).

Parity status: every function here is pinned by tests/test_oracle_pins.py
(page worked example, closed forms, special cases and library cross-checks).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Callable, Iterable, Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "engram_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle_engram.so")

F32, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(_LIB_DIR, exist_ok=True)
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        P = C.c_void_p
        i32, i64, dbl = C.c_int, C.c_int64, C.c_double
        sig = {
            "oracle_widen": (None, [P, i64, i32, P]),
            "oracle_compress_ids": (None, [P, i64, P, P]),
            "oracle_shifted_token": (i64, [P, i32, i32, i32, i32, P, i32, i64]),
            "oracle_shift": (None, [P, i32, i32, i32, P, i32, i64, P]),
            "oracle_hash": (None, [P, i32, i32, P, i32, i32, P, i32, P, P, i64, P]),
            "oracle_gather": (None, [P, i32, i32, P, P, i64, i32, P]),
            "oracle_gate_value": (dbl, [dbl, dbl]),
            "oracle_token_gate": (None, [P, i32, i32, i32, P, P, P, P, i32, P, i64, i32,
                                         dbl, dbl, P, P, P, P]),
            "oracle_tokens_gate": (None, [P, i64, i32, i32, i32, P, P, P, P, i32, P, i32,
                                          dbl, dbl, P, P, P, P, i32]),
            "oracle_rmsnorm": (None, [P, i32, P, dbl, P]),
            "oracle_conv_point": (None, [P, P, P, i32, i32, i32, P, i32, P]),
            "oracle_short_conv": (None, [P, i32, i32, i32, P, i32, i32, P, P]),
            "oracle_forward": (None, [P, i32, i32, i32, P, i32, i32, P, P, P, i64,
                                      P, P, P, P, P, P, P, i32, i32, i32, i32, i32,
                                      dbl, dbl, P, P, P, P, P, P, i32]),
        }
        for name, (res, args) in sig.items():
            f = getattr(_lib, name)
            f.restype = res
            f.argtypes = args
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _i64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def storage(t) -> Tuple[np.ndarray, int]:
    """(contiguous host array, storage code) for a float32 or bfloat16 tensor.
    bfloat16 is carried as its raw 16-bit pattern."""
    import torch
    if isinstance(t, np.ndarray):
        if t.dtype == np.float32:
            return np.ascontiguousarray(t), F32
        if t.dtype == np.uint16:
            return np.ascontiguousarray(t), BF16
        raise TypeError(t.dtype)
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.float32:
        return t.numpy(), F32
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), BF16
    raise TypeError(t.dtype)


def widen(a: np.ndarray, code: int) -> np.ndarray:
    out = np.empty(a.size, dtype=np.float64)
    lib().oracle_widen(_p(a), a.size, code, _p(out))
    return out.reshape(a.shape)


# ---- steps ----------------------------------------------------------------

def compress_ids(raw, lookup) -> np.ndarray:
    raw, lookup = _i64(raw), _i64(lookup)
    out = np.empty_like(raw)
    lib().oracle_compress_ids(_p(raw), raw.size, _p(lookup), _p(out))
    return out


def shift(x, k: int, pad_id: int, hist=None) -> np.ndarray:
    x = _i64(x)
    B, T = x.shape
    h = None if hist is None else _i64(hist)
    out = np.empty_like(x)
    lib().oracle_shift(_p(x), B, T, k, _p(h), 0 if h is None else h.shape[1], pad_id, _p(out))
    return out


def ngram_hash(x, orders: Sequence[int], J: int, mult, primes, pad_id: int,
               hist=None) -> np.ndarray:
    """idx [B, T, len(orders)*J] (int64)."""
    x = _i64(x)
    B, T = x.shape
    o = np.ascontiguousarray(np.asarray(orders, dtype=np.int32))
    m, p = _i64(mult), _i64(primes)
    h = None if hist is None else _i64(hist)
    nh = len(orders) * J
    idx = np.empty((B, T, nh), dtype=np.int64)
    lib().oracle_hash(_p(x), B, T, _p(h), 0 if h is None else h.shape[1], len(orders),
                      _p(o), J, _p(m), _p(p), pad_id, _p(idx))
    return idx


def gather(table: np.ndarray, row_offsets, idx) -> np.ndarray:
    """e [M, nh*Dh] in the table's storage dtype (a byte copy of the rows)."""
    idx = _i64(idx)
    nh = idx.shape[-1]
    M = idx.size // nh
    Dh = table.shape[1]
    off = _i64(row_offsets)
    e = np.empty((M, nh * Dh), dtype=table.dtype)
    lib().oracle_gather(_p(table), table.dtype.itemsize, Dh, _p(off), _p(idx), M, nh, _p(e))
    return e


def gate_value(s: float, gate_eps: float = 1e-6) -> float:
    return lib().oracle_gate_value(float(s), float(gate_eps))


def rmsnorm(x, w, eps: float) -> np.ndarray:
    x, w = _f64(x), _f64(w)
    out = np.empty_like(x)
    lib().oracle_rmsnorm(_p(x), x.size, _p(w), eps, _p(out))
    return out


def tokens_gate(e: np.ndarray, H: int, hc: int, w_value, w_key, norm_key, norm_query,
                hidden, rms_eps: float, gate_eps: float, nthreads: int = 0):
    """For n tokens: V [n, H], s [n, hc], g [n, hc] (float64).
    e: [n, E] float64; hidden: [n, hc, H] storage; weights: storage tensors."""
    e = _f64(e)
    n, E = e.shape
    wv, code = storage(w_value)
    wk, c2 = storage(w_key)
    nk, c3 = storage(norm_key)
    nq, c4 = storage(norm_query)
    hs, hcode = storage(hidden)
    assert code == c2 == c3 == c4
    nthreads = nthreads or (os.cpu_count() or 1)
    V = np.empty((n, H))
    s = np.empty((n, hc))
    g = np.empty((n, hc))
    work = np.empty(nthreads * 6 * H)
    lib().oracle_tokens_gate(_p(e), n, E, H, hc, _p(wv), _p(wk), _p(nk), _p(nq), code,
                             _p(hs), hcode, rms_eps, gate_eps, _p(V), _p(s), _p(g),
                             _p(work), nthreads)
    return V, s, g


def conv_point(Vtap: np.ndarray, gtap: np.ndarray, valid: np.ndarray, conv_w) -> np.ndarray:
    """Y [hc, H] at one position from its K taps (oldest first)."""
    Vtap, gtap = _f64(Vtap), _f64(gtap)
    K, H = Vtap.shape
    hc = gtap.shape[1]
    v = np.ascontiguousarray(np.asarray(valid, dtype=np.int32))
    cw, code = storage(conv_w)
    Y = np.empty((hc, H))
    lib().oracle_conv_point(_p(Vtap), _p(gtap), _p(v), K, H, hc, _p(cw), code, _p(Y))
    return Y


def short_conv(U, conv_w, K: int, dil: int, prev=None) -> np.ndarray:
    """Y = U + causal depthwise dilated conv(U); U [B, T, C] float64, conv_w [C, K]."""
    U = _f64(U)
    B, T, Cc = U.shape
    w = _f64(conv_w)
    pv = None if prev is None else _f64(prev)
    Y = np.empty_like(U)
    lib().oracle_short_conv(_p(U), B, T, Cc, _p(w), K, dil, _p(pv), _p(Y))
    return Y


# ---- whole pass -----------------------------------------------------------

def forward(x, orders, J, mult, primes, row_offsets, pad_id, table, w_value, w_key,
            norm_key, norm_query, conv_w, hidden, K: int, dil: int,
            rms_eps: float = 1e-6, gate_eps: float = 1e-6, nthreads: int = 0):
    """Whole forward with host inputs.  x: compressed ids [B, T];
    hidden [B, T, hc, H].  Returns dict of float64 arrays Y, V, s, g and idx."""
    x = _i64(x)
    B, T = x.shape
    tb, code = storage(table)
    Dh = tb.shape[1]
    arrs = [storage(a) for a in (w_value, w_key, norm_key, norm_query, conv_w, hidden)]
    assert all(c == code for _, c in arrs), "all tensors must share one storage type"
    wv, wk, nk, nq, cw, hs = [a for a, _ in arrs]
    hc, H = hs.shape[-2], hs.shape[-1]
    nh = len(orders) * J
    E = nh * Dh
    M = B * T
    nthreads = nthreads or (os.cpu_count() or 1)
    o = np.ascontiguousarray(np.asarray(orders, dtype=np.int32))
    m, p, off = _i64(mult), _i64(primes), _i64(row_offsets)
    Y = np.empty((B, T, hc, H))
    idx = np.empty((B, T, nh), dtype=np.int64)
    V = np.empty((B, T, H))
    s = np.empty((B, T, hc))
    g = np.empty((B, T, hc))
    work = np.empty(M * (nh + H + 2 * hc) + nthreads * (E + 6 * H))
    lib().oracle_forward(_p(x), B, T, len(orders), _p(o), J, Dh, _p(m), _p(p), _p(off),
                         pad_id, _p(tb), _p(wv), _p(wk), _p(nk), _p(nq), _p(cw), _p(hs),
                         code, H, hc, K, dil, rms_eps, gate_eps, _p(Y), _p(idx), _p(V),
                         _p(s), _p(g), _p(work), nthreads)
    return {"Y": Y, "idx": idx, "V": V, "s": s, "g": g}


def forward_sampled(x, positions: Iterable[Tuple[int, int]], orders, J, mult, primes,
                    row_offsets, pad_id, fetch_rows: Callable[[np.ndarray], object],
                    fetch_hidden: Callable[[np.ndarray, np.ndarray], object],
                    w_value, w_key, norm_key, norm_query, conv_w, K: int, dil: int,
                    rms_eps: float = 1e-6, gate_eps: float = 1e-6, nthreads: int = 0):
    """Y at the given (b, t) positions of the prefill over x [B, T].

    fetch_rows(rows [n]) -> storage tensor [n, Dh] of table rows;
    fetch_hidden(b [n], t [n]) -> storage tensor [n, hc, H].
    Returns (Y [P, hc, H], s [P, hc], g [P, hc], idx [B, T, nh]) where s, g are
    those of the sampled positions themselves."""
    x = _i64(x)
    B, T = x.shape
    pos = [(int(b), int(t)) for b, t in positions]
    idx = ngram_hash(x, orders, J, mult, primes, pad_id)
    nh = idx.shape[-1]
    need = sorted({(b, t - (K - 1 - i) * dil) for b, t in pos for i in range(K)
                   if t - (K - 1 - i) * dil >= 0})
    where = {bt: n for n, bt in enumerate(need)}
    nb = np.array([b for b, _ in need], dtype=np.int64)
    nt = np.array([t for _, t in need], dtype=np.int64)
    rows = (np.asarray(row_offsets, dtype=np.int64)[None, :] + idx[nb, nt, :]).reshape(-1)
    rs, rcode = storage(fetch_rows(rows))
    Dh = rs.shape[1]
    e = widen(rs, rcode).reshape(len(need), nh * Dh)
    hs = fetch_hidden(nb, nt)
    H = storage(w_value)[0].shape[0]
    hc = storage(norm_key)[0].shape[0]
    V, s, g = tokens_gate(e, H, hc, w_value, w_key, norm_key, norm_query, hs,
                          rms_eps, gate_eps, nthreads)
    Y = np.empty((len(pos), hc, H))
    s_out = np.empty((len(pos), hc))
    g_out = np.empty((len(pos), hc))
    for n, (b, t) in enumerate(pos):
        Vtap = np.zeros((K, H))
        gtap = np.zeros((K, hc))
        valid = np.zeros(K, dtype=np.int32)
        for i in range(K):
            tp = t - (K - 1 - i) * dil
            if tp >= 0:
                j = where[(b, tp)]
                Vtap[i], gtap[i], valid[i] = V[j], g[j], 1
        Y[n] = conv_point(Vtap, gtap, valid, conv_w)
        j = where[(b, t)]
        s_out[n], g_out[n] = s[j], g[j]
    return Y, s_out, g_out, idx


# ---- a table sharded over R devices ---------------------------------------
# The explainer page (§4.4, system efficiency) shards the tables across GPUs in
# training and collects the active rows with an All-to-All; it fixes no split.
# Reading used here: shard r of R holds the stacked table's rows r, r+R, r+2R,
# ... (row -> shard row % R, local row row // R), so that every head's rows
# and every skewed id spread evenly over the shards.

def shard_table(table: np.ndarray, n_shards: int, r: int) -> np.ndarray:
    """Shard r of n_shards: rows r, r + n_shards, ... of the stacked table."""
    return np.ascontiguousarray(table[r::n_shards])


def shard_route(rows, n_shards: int) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Requests of the sharded gather of absolute rows ``rows`` (one per row q
    of e, q = m*nh + h, in that order).  Returns (counts [R], req_rows [N],
    req_pos [N]): the requests grouped by shard (shard 0 first), in increasing
    q within a shard; request k asks its shard for local row req_rows[k] and
    fills row req_pos[k] of e; counts[r] requests go to shard r."""
    rows = _i64(rows).reshape(-1)
    owner = rows % n_shards
    order = np.argsort(owner, kind="stable")      # group by shard, q order kept
    counts = np.bincount(owner, minlength=n_shards).astype(np.int64)
    return counts, (rows // n_shards)[order], order.astype(np.int32)
