"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
oracle run on the same inputs (whole pass, or sampled positions with rows
fetched from the device tables), and the tolerance rule.

Tolerance (the bound set for this pass, per output tensor): max |y - y_ref| must not
exceed tol * max |y_ref| with tol = 1e-4 for float32 and 2e-2 for bfloat16,
y_ref from the float64 oracle on the same (bf16-valued) inputs.
"""
from __future__ import annotations

import numpy as np
import torch

from hashed_gram_conditional_hash_b200 import workloads as W
from oracle import engram_oracle as O

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


def oracle_ids(p) -> np.ndarray:
    x = p.ids.cpu().numpy()
    if p.lookup is not None:
        x = O.compress_ids(x, p.lookup.cpu().numpy())
    return x


def oracle_forward_full(p, conv_w=None):
    w = p.w
    return O.forward(x=oracle_ids(p), orders=w.orders, J=w.heads_per_order, mult=p.mult,
                     primes=p.primes, row_offsets=p.offsets, pad_id=w.pad_id,
                     table=p.table.cpu(), w_value=p.w_value.cpu(), w_key=p.w_key.cpu(),
                     norm_key=p.norm_key.cpu(), norm_query=p.norm_query.cpu(),
                     conv_w=(p.conv_w if conv_w is None else conv_w).cpu(),
                     hidden=p.hidden.cpu(), K=w.conv_kernel, dil=w.dil,
                     rms_eps=w.rms_eps, gate_eps=w.gate_eps)


def oracle_at(p, positions, hidden_bt=None, x=None):
    """Oracle Y (and s, g) at (b, t) positions.  hidden_bt(b, t) -> [n, hc, H]
    (default: p.hidden[b, t]); x: compressed ids [B, T] (default: p.ids)."""
    w = p.w
    dev = p.table.device
    if hidden_bt is None:
        hidden_bt = lambda b, t: p.hidden[torch.from_numpy(b).to(dev), torch.from_numpy(t).to(dev)]
    if x is None:
        x = oracle_ids(p)
    fetch_rows = lambda r: p.table[torch.from_numpy(r).to(dev)].cpu()
    fetch_hidden = lambda b, t: hidden_bt(b, t).cpu()
    return O.forward_sampled(x, positions, w.orders, w.heads_per_order, p.mult, p.primes,
                             p.offsets, w.pad_id, fetch_rows, fetch_hidden, p.w_value.cpu(),
                             p.w_key.cpu(), p.norm_key.cpu(), p.norm_query.cpu(),
                             p.conv_w.cpu(), K=w.conv_kernel, dil=w.dil,
                             rms_eps=w.rms_eps, gate_eps=w.gate_eps)


def sample_positions(B: int, T: int, dil: int, n_random: int, seed: int = 0):
    """Edges of every sequence that are special for the shift and the conv
    (t < (K-1)*dil, the last positions) plus random interior positions."""
    rng = np.random.default_rng(seed)
    edge_t = sorted({t for t in (0, 1, 2, dil - 1, dil, 2 * dil, 3 * dil - 1, 3 * dil,
                                 T // 2, T - 2, T - 1) if 0 <= t < T})
    bs = sorted({0, B - 1, B // 2})
    pos = [(b, t) for b in bs for t in edge_t]
    for _ in range(n_random):
        pos.append((int(rng.integers(0, B)), int(rng.integers(0, T))))
    return sorted(set(pos))


def device_params(w: W.Workload, device="cuda"):
    return W.make_params(w, device)


def make_layer(p, table=None):
    """EngramLayer of a workloads.Params (table: another copy of the table)."""
    from hashed_gram_conditional_hash_b200 import EngramLayer
    w = p.w
    return EngramLayer(orders=w.orders, heads_per_order=w.heads_per_order, row_dim=w.row_dim,
                       hidden=w.hidden, hc_mult=w.hc_mult, conv_kernel=w.conv_kernel,
                       dilation=w.dil, pad_id=w.pad_id, vocab=w.vocab,
                       table=p.table if table is None else table, row_offsets=p.offsets,
                       primes=p.primes, multipliers=p.mult, w_value=p.w_value, w_key=p.w_key,
                       norm_key=p.norm_key, norm_query=p.norm_query, conv_w=p.conv_w,
                       lookup=p.lookup, rms_eps=w.rms_eps, gate_eps=w.gate_eps)
