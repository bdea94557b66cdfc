"""Seeded synthetic inputs for the Engram forward pass.

This module only *draws* inputs: token streams, the compressed-ID lookup, the
per-layer odd multipliers, the per-head prime moduli and the random tensors
(tables, projections, norms, conv taps, hidden states).  It performs none of
the method's arithmetic (no hashing, gathering, projection, gating or
convolution); both the CUDA path and the CPU oracle consume what it returns.

Shapes and distributions follow the five workloads the Engram pages are
benchmarked on here:

* tiny fp32        B=1,  T=128,  raw vocab 2048 -> 1580 compressed IDs, uniform
* model bf16       B=4,  T=2048, vocab 98,304, Zipf(1.1)
* large-table bf16 B=8,  T=4096, vocab 128,000, Zipf(1.05), ~3.2 GB of tables
* HBM-table bf16   B=16, T=4096, vocab 128,000, 50% Zipf(1.0) + 50% uniform,
                   ~17.2 GB of tables
* decode bf16      1024 sequences x 1 token per call x 256 calls

Parameter drawing follows the Engram formulas page: multipliers are odd,
m = 2r + 1 with r < 2^30, drawn from a per-layer seed
seed_layer = seed + PRIME_1 * layer_id (formulas page §1.2 parameter list and
§1.4, where the operator between ``seed`` and ``PRIME_1`` is lost in the text and
is read here as ``+``); every (order, head) gets its own prime modulus
(formulas page §1.2 step 2, §1.4; explainer page §2.2 1)), taken here as the
ascending run of primes starting at the workload's base.
"""
from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np
import torch

#: Odd constant that separates per-layer multiplier seeds.  The formulas page
#: names PRIME_1 but prints no value; any fixed prime serves.
PRIME_1 = 10007


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    orders: Tuple[int, ...]
    heads_per_order: int
    row_dim: int
    hidden: int
    hc_mult: int
    dtype: str                       # "f32" | "bf16"
    vocab: int                       # compressed vocabulary size
    token_dist: str = "uniform"      # "uniform" | "zipf" | "mix"
    zipf_s: float = 1.0
    raw_vocab: Optional[int] = None  # set -> ids are raw and go through a lookup
    prime_base: int = 1009
    pad_id: int = 0
    conv_kernel: int = 4
    dilation: Optional[int] = None   # default: max n-gram order
    seed: int = 0
    layer_id: int = 0
    decode_calls: int = 0            # >0: T must be 1; stream of this many calls
    norm_w_std: float = 0.0          # 0 -> RMSNorm weights are exactly 1
    table_std: float = 0.02
    w_std: Optional[float] = None    # default 1/sqrt(E)
    hidden_std: float = 1.0
    conv_std: float = 0.1
    rms_eps: float = 1e-6
    gate_eps: float = 1e-6

    # ---- derived sizes -------------------------------------------------
    @property
    def max_n(self) -> int:
        return max(self.orders)

    @property
    def n_hist(self) -> int:
        return self.max_n - 1

    @property
    def dil(self) -> int:
        return self.dilation if self.dilation is not None else self.max_n

    @property
    def nh(self) -> int:
        return len(self.orders) * self.heads_per_order

    @property
    def E(self) -> int:
        return self.nh * self.row_dim

    @property
    def M(self) -> int:
        return self.B * self.T

    @property
    def seq_len(self) -> int:
        """Length of each token stream (decode: number of calls)."""
        return self.decode_calls if self.decode_calls else self.T

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


CONFIGS: Dict[str, Workload] = {
    "tiny_f32": Workload(
        name="tiny_f32", B=1, T=128, orders=(2, 3), heads_per_order=4, row_dim=32,
        hidden=256, hc_mult=1, dtype="f32", vocab=1580, raw_vocab=2048,
        token_dist="uniform", prime_base=1009, pad_id=0, dilation=3, seed=1000),
    "model_bf16": Workload(
        name="model_bf16", B=4, T=2048, orders=(2, 3), heads_per_order=8, row_dim=64,
        hidden=1024, hc_mult=4, dtype="bf16", vocab=98_304, token_dist="zipf",
        zipf_s=1.1, prime_base=65_536, dilation=3, seed=1001),
    "large_table_bf16": Workload(
        name="large_table_bf16", B=8, T=4096, orders=(2, 3, 4), heads_per_order=8,
        row_dim=64, hidden=2560, hc_mult=4, dtype="bf16", vocab=128_000,
        token_dist="zipf", zipf_s=1.05, prime_base=1 << 20, dilation=4, seed=1002),
    "hbm_table_bf16": Workload(
        name="hbm_table_bf16", B=16, T=4096, orders=(2, 3), heads_per_order=16,
        row_dim=64, hidden=4096, hc_mult=4, dtype="bf16", vocab=128_000,
        token_dist="mix", zipf_s=1.0, prime_base=1 << 22, dilation=3, seed=1003),
    "decode_bf16": Workload(
        name="decode_bf16", B=1024, T=1, orders=(2, 3, 4), heads_per_order=8,
        row_dim=64, hidden=2048, hc_mult=4, dtype="bf16", vocab=98_304,
        token_dist="zipf", zipf_s=1.1, prime_base=1 << 20, dilation=4, seed=1004,
        decode_calls=256),
}


# ---- parameter draws ------------------------------------------------------

def _is_prime(n: int) -> bool:
    if n < 2:
        return False
    if n % 2 == 0:
        return n == 2
    f = 3
    while f * f <= n:
        if n % f == 0:
            return False
        f += 2
    return True


def primes_from(base: int, count: int) -> np.ndarray:
    """The ``count`` smallest primes >= ``base``, ascending (all distinct)."""
    out = []
    n = max(2, base)
    while len(out) < count:
        if _is_prime(n):
            out.append(n)
        n += 1
    return np.asarray(out, dtype=np.int64)


def head_primes(w: Workload) -> np.ndarray:
    """One prime per (order, head), in (order ascending, head ascending) order."""
    return primes_from(w.prime_base, w.nh)


def row_offsets(primes: np.ndarray) -> np.ndarray:
    """First row of each (order, head) table inside the stacked table."""
    return np.concatenate([[0], np.cumsum(primes)[:-1]]).astype(np.int64)


def multipliers(w: Workload) -> np.ndarray:
    """Odd per-layer multipliers m_k = 2 r_k + 1, r_k uniform in [0, 2^30)."""
    rng = np.random.default_rng(w.seed + PRIME_1 * w.layer_id)
    r = rng.integers(0, 1 << 30, size=w.max_n, dtype=np.int64)
    return (r * 2 + 1).astype(np.int64)


def compress_lookup(w: Workload) -> Optional[np.ndarray]:
    """Surjective raw -> compressed lookup standing in for the normalised
    tokenizer vocabulary: a seeded permutation covers every compressed ID with
    the first ``vocab`` raw IDs, the remaining raw IDs fold onto random ones."""
    if w.raw_vocab is None:
        return None
    rng = np.random.default_rng([w.seed, 11])
    lut = np.empty(w.raw_vocab, dtype=np.int64)
    lut[: w.vocab] = rng.permutation(w.vocab)
    lut[w.vocab:] = rng.integers(0, w.vocab, size=w.raw_vocab - w.vocab)
    return lut


def _zipf_ids(rng: np.random.Generator, vocab: int, s: float, n: int) -> np.ndarray:
    ranks = np.arange(1, vocab + 1, dtype=np.float64)
    cdf = np.cumsum(ranks ** (-s))
    cdf /= cdf[-1]
    r = np.searchsorted(cdf, rng.random(n), side="right")
    r = np.minimum(r, vocab - 1)
    rank_to_id = rng.permutation(vocab)
    return rank_to_id[r].astype(np.int64)


def token_ids(w: Workload) -> np.ndarray:
    """Token stream [B, seq_len] (raw IDs when the workload has a raw vocab)."""
    rng = np.random.default_rng([w.seed, 1])
    n = w.B * w.seq_len
    if w.raw_vocab is not None:
        ids = rng.integers(0, w.raw_vocab, size=n, dtype=np.int64)
    elif w.token_dist == "uniform":
        ids = rng.integers(0, w.vocab, size=n, dtype=np.int64)
    elif w.token_dist == "zipf":
        ids = _zipf_ids(rng, w.vocab, w.zipf_s, n)
    elif w.token_dist == "mix":
        z = _zipf_ids(rng, w.vocab, w.zipf_s, n)
        u = rng.integers(0, w.vocab, size=n, dtype=np.int64)
        coin = rng.random(n) < 0.5
        ids = np.where(coin, z, u)
    else:
        raise ValueError(w.token_dist)
    return ids.reshape(w.B, w.seq_len)


# ---- tensors --------------------------------------------------------------

def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std: float, mean: float, dtype, device, seed: int) -> torch.Tensor:
    t = torch.empty(shape, dtype=dtype, device=device)
    t.normal_(mean, std, generator=_gen(device, seed))
    return t


def table_bytes(w: Workload) -> int:
    return int(head_primes(w).sum()) * w.row_dim * w.elem_bytes


def gen_device_for(w: Workload, device: str) -> str:
    """Small tensors are drawn on the CPU (identical on every machine); tables
    above 1 GiB are drawn directly on the target device."""
    return device if (table_bytes(w) > (1 << 30) and device != "cpu") else "cpu"


@dataclass
class Params:
    """Every input of one Engram layer (torch tensors on ``device``)."""
    w: Workload
    ids: torch.Tensor          # int64 [B, seq_len]  (raw when lookup is set)
    lookup: Optional[torch.Tensor]
    primes: np.ndarray         # int64 [nh]   (host)
    offsets: np.ndarray        # int64 [nh]   (host)
    mult: np.ndarray           # int64 [max_n] (host)
    table: torch.Tensor        # [total_rows, row_dim]
    w_value: torch.Tensor      # [H, E]
    w_key: torch.Tensor        # [hc, H, E]
    norm_key: torch.Tensor     # [hc, H]
    norm_query: torch.Tensor   # [hc, H]
    conv_w: torch.Tensor       # [hc*H, K]
    hidden: torch.Tensor       # [B, T, hc, H]; decode: [calls, B, hc, H]
    gen_device: str = "cpu"


def make_params(w: Workload, device: str = "cpu", with_hidden: bool = True) -> Params:
    gdev = gen_device_for(w, device)
    dt = w.torch_dtype
    primes = head_primes(w)
    offs = row_offsets(primes)
    total_rows = int(primes.sum())
    s = w.seed * 100
    table = _normal((total_rows, w.row_dim), w.table_std, 0.0, dt, gdev, s + 2)
    wstd = w.w_std if w.w_std is not None else 1.0 / math.sqrt(w.E)
    w_value = _normal((w.hidden, w.E), wstd, 0.0, dt, gdev, s + 3)
    w_key = _normal((w.hc_mult, w.hidden, w.E), wstd, 0.0, dt, gdev, s + 4)
    if w.norm_w_std > 0:
        nk = _normal((w.hc_mult, w.hidden), w.norm_w_std, 1.0, dt, gdev, s + 5)
        nq = _normal((w.hc_mult, w.hidden), w.norm_w_std, 1.0, dt, gdev, s + 6)
    else:
        nk = torch.ones((w.hc_mult, w.hidden), dtype=dt, device=gdev)
        nq = torch.ones((w.hc_mult, w.hidden), dtype=dt, device=gdev)
    conv_w = _normal((w.hc_mult * w.hidden, w.conv_kernel), w.conv_std, 0.0, dt, gdev, s + 7)
    if with_hidden:
        if w.decode_calls:
            hshape = (w.decode_calls, w.B, w.hc_mult, w.hidden)
        else:
            hshape = (w.B, w.T, w.hc_mult, w.hidden)
        hidden = _normal(hshape, w.hidden_std, 0.0, dt, gdev, s + 8)
    else:
        hidden = torch.empty(0, dtype=dt)
    ids = torch.from_numpy(token_ids(w))
    lut = compress_lookup(w)
    lookup = torch.from_numpy(lut) if lut is not None else None

    def mv(t):
        return t.to(device) if t is not None else None

    return Params(w=w, ids=mv(ids), lookup=mv(lookup), primes=primes, offsets=offs,
                  mult=multipliers(w), table=mv(table), w_value=mv(w_value),
                  w_key=mv(w_key), norm_key=mv(nk), norm_query=mv(nq),
                  conv_w=mv(conv_w), hidden=mv(hidden), gen_device=gdev)


def small_workload(**kw) -> Workload:
    """A few-tile test shape (ragged tails on every axis unless overridden)."""
    base = dict(name="small", B=3, T=77, orders=(2, 3), heads_per_order=2, row_dim=64,
                hidden=256, hc_mult=2, dtype="bf16", vocab=5000, token_dist="zipf",
                zipf_s=1.1, prime_base=3001, dilation=3, seed=7, norm_w_std=0.1)
    base.update(kw)
    return Workload(**base)
