"""The C-ABI library loads on a machine without a GPU, exports every function
include/engram.h declares, and rejects bad arguments on the host before any
launch (no compute calls here)."""
import ctypes as C
import os
import re

import pytest
import torch

from hashed_gram_conditional_hash_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "engram.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(engram_\w+)\s*\(", src)))


def test_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 13
    lib = C.CDLL(L.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_error_text():
    assert L.engram_version() >= 100
    cfg = L.make_config((2, 3), 4, 32, 256, 1, 4, 3, 0, 1580, torch.float32)
    cfg.n_orders = 0
    n = C.c_size_t(0)
    assert L.lib().engram_forward_workspace_size(C.byref(cfg), 1, 8, C.byref(n)) == 1
    assert "n_orders" in L.last_error()


def _cfg(**kw):
    c = L.make_config((2, 3), 2, 64, 256, 2, 4, 3, 0, 5000, torch.bfloat16)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value", [
    ("heads_per_order", 0), ("heads_per_order", 40), ("hc_mult", 9), ("conv_kernel", 0),
    ("dilation", 0), ("pad_id", -1), ("pad_id", 1 << 32), ("vocab", 0), ("rms_eps", 0.0),
    ("dtype", 7)])
def test_config_validation(field, value):
    n = C.c_size_t(0)
    cfg = _cfg(**{field: value})
    assert L.lib().engram_forward_workspace_size(C.byref(cfg), 2, 8, C.byref(n)) == 1


def test_orders_must_ascend():
    cfg = _cfg()
    cfg.orders[1] = 2
    n = C.c_size_t(0)
    assert L.lib().engram_forward_workspace_size(C.byref(cfg), 2, 8, C.byref(n)) == 1


@pytest.mark.parametrize("mult,primes", [
    ([2, 3, 5], [101] * 4),               # even multiplier
    ([1 << 31, 3, 5], [101] * 4),         # multiplier too large
    ([1, 3, 5], [1, 101, 103, 107]),      # modulus < 2
    ([1, 3, 5], [1 << 31, 101, 103, 107]),
])
def test_hash_parameter_validation(mult, primes):
    cfg = _cfg()
    m = (C.c_int64 * 3)(*mult)
    p = (C.c_int64 * 4)(*primes)
    # pointers are never dereferenced: the call fails on the host first
    rc = L.lib().engram_hash(C.byref(cfg), C.c_void_p(16), 1, 4, None, m, p, C.c_void_p(16),
                             None, None)
    assert rc == 1


def test_workspace_sizes_grow_with_tokens():
    cfg = _cfg()
    a = L.engram_forward_workspace_size(cfg, 1, 128)
    b = L.engram_forward_workspace_size(cfg, 4, 128)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    assert L.engram_gate_fuse_workspace_size(cfg, 512) > 0


def test_forward_rejects_null_and_misaligned():
    cfg = _cfg()
    w = L.EngramWeights()
    ws_n = L.engram_forward_workspace_size(cfg, 1, 4)
    rc = L.lib().engram_forward(C.byref(cfg), C.byref(w), C.c_void_p(256), 1, 4, C.c_void_p(256),
                                C.c_void_p(256), None, C.c_void_p(256), ws_n, None, None)
    assert rc == 1 and "NULL" in L.last_error()
    for f in ("table", "w_value", "w_key", "norm_key", "norm_query", "conv_w"):
        setattr(w, f, 4096)
    w.table = 4100  # not 16-byte aligned
    rc = L.lib().engram_forward(C.byref(cfg), C.byref(w), C.c_void_p(256), 1, 4, C.c_void_p(256),
                                C.c_void_p(256), None, C.c_void_p(256), ws_n, None, None)
    assert rc == 1 and "aligned" in L.last_error()


def test_row_count_above_2_30_is_unsupported_before_any_pointer_is_read():
    # B*T*heads above 2^30: the kernels index (token, head) rows in 32 bits, so
    # the forward, the gathers and the forward from gathered rows refuse the
    # call on the host (the pointers below are never dereferenced)
    cfg = _cfg()                                           # 2 orders x 2 heads
    w = L.EngramWeights()
    B, T = 1 << 14, 1 << 15                                 # 2^29 tokens x 4 heads = 2^31 rows
    rc = L.lib().engram_forward(C.byref(cfg), C.byref(w), C.c_void_p(256), B, T, C.c_void_p(256),
                                C.c_void_p(256), None, C.c_void_p(256), 0, None, None)
    assert rc == 2 and "2^30" in L.last_error()
    rc = L.lib().engram_gather_ids(C.byref(cfg), C.byref(w), C.c_void_p(256), B, T, None, C.c_void_p(256),
                                   None, None)
    assert rc == 2 and "2^30" in L.last_error()
    rc = L.lib().engram_forward_gathered(C.byref(cfg), C.byref(w), C.c_void_p(256), B, T, C.c_void_p(256),
                                         C.c_void_p(256), C.c_void_p(256), 0, None, None)
    assert rc == 2 and "2^30" in L.last_error()
    # 2^30 rows exactly is accepted by the count check (the null weights fail later)
    rc = L.lib().engram_gather_ids(C.byref(cfg), C.byref(w), C.c_void_p(256), 1 << 14, 1 << 14, None,
                                   C.c_void_p(256), None, None)
    assert "2^30" not in L.last_error()


def test_short_conv_rejects_aliasing():
    cfg = _cfg()
    rc = L.lib().engram_short_conv(C.byref(cfg), C.c_void_p(256), 1, 4, C.c_void_p(512), None,
                                   C.c_void_p(256), None)
    assert rc == 1


# ---- the split pass, several layers and the sharded table: host-side checks
P = C.c_void_p


def _weights():
    w = L.EngramWeights()
    w.table = 256
    w.total_rows = 1000
    return w


def test_gather_ids_layers_rejects_layer_counts():
    cfg = _cfg()
    w = _weights()
    arr = (C.POINTER(L.EngramWeights) * 1)(C.pointer(w))
    e = (P * 1)(256)
    for n in (0, L.MAX_LAYERS + 1):
        assert L.lib().engram_gather_ids_layers(C.byref(cfg), arr, n, P(256), 2, 8, None, e, None, None) == 1
        assert "n_layers" in L.last_error()
    assert L.lib().engram_gather_ids_layers(C.byref(cfg), None, 1, P(256), 2, 8, None, e, None, None) == 1


@pytest.mark.parametrize("n_shards", [0, L.MAX_SHARDS + 1])
def test_shard_route_rejects_shard_counts(n_shards):
    cfg = _cfg()
    w = _weights()
    rc = L.lib().engram_shard_route(C.byref(cfg), C.byref(w), P(256), 2, 8, None, n_shards, P(256), P(256),
                                    P(256), P(256), 1 << 20, None, None)
    assert rc == 1 and "n_shards" in L.last_error()


def test_shard_route_rejects_missing_or_small_workspace():
    cfg = _cfg()
    w = _weights()
    need = L.engram_shard_route_workspace_size(cfg, 2, 8, 4)
    assert need > 0
    args = lambda counts, ws, nbytes: (C.byref(cfg), C.byref(w), P(256), 2, 8, None, 4, counts, P(256), P(256),
                                       ws, nbytes, None, None)
    assert L.lib().engram_shard_route(*args(None, P(256), need)) == 1          # counts NULL
    assert L.lib().engram_shard_route(*args(P(256), None, need)) == 1          # ws NULL
    assert L.lib().engram_shard_route(*args(P(256), P(272), need)) == 1        # ws not 256-byte aligned
    assert "aligned" in L.last_error()
    assert L.lib().engram_shard_route(*args(P(256), P(256), need - 1)) == 1    # too small
    assert "too small" in L.last_error()
    big = _cfg(heads_per_order=32)                                            # B*T*nh >= 2^31
    assert L.lib().engram_shard_route(C.byref(big), C.byref(w), P(256), 1 << 20, 1 << 10, None, 2, P(256),
                                      P(256), P(256), P(256), 1 << 20, None, None) == 2


def test_shard_serve_and_place_reject_bad_arguments():
    cfg = _cfg()
    lib = L.lib()
    assert lib.engram_shard_serve(C.byref(cfg), P(256), 10, P(256), -1, P(256), None, None) == 1
    assert lib.engram_shard_serve(C.byref(cfg), None, 10, P(256), 4, P(256), None, None) == 1
    assert lib.engram_shard_serve(C.byref(cfg), P(256), 10, P(256), 4, P(264), None, None) == 1   # misaligned out
    narrow = _cfg(row_dim=2)                                                  # 4-byte rows
    assert lib.engram_shard_serve(C.byref(narrow), P(256), 10, P(256), 4, P(256), None, None) == 2
    assert lib.engram_shard_place(C.byref(cfg), P(256), P(256), -1, P(256), 8, None, None) == 1
    assert lib.engram_shard_place(C.byref(cfg), P(256), None, 4, P(256), 8, None, None) == 1
    assert lib.engram_shard_place(C.byref(cfg), P(264), P(256), 4, P(256), 8, None, None) == 1    # misaligned got
    assert lib.engram_shard_place(C.byref(narrow), P(256), P(256), 4, P(256), 8, None, None) == 2
    # nothing to do is not an error, and launches nothing
    assert lib.engram_shard_serve(C.byref(cfg), None, 0, None, 0, None, None, None) == 0
    assert lib.engram_shard_place(C.byref(cfg), None, None, 0, None, 0, None, None) == 0


def test_forward_gathered_rejects_null_misaligned_and_small_workspace():
    cfg = _cfg()
    w = L.EngramWeights()
    for f in ("w_value", "w_key", "norm_key", "norm_query", "conv_w"):
        setattr(w, f, 256)
    need = L.engram_forward_workspace_size(cfg, 2, 8)
    lib = L.lib()
    ok = dict(e=P(256), hidden=P(256), y=P(256), ws=P(256), n=need)
    call = lambda **kw: lib.engram_forward_gathered(C.byref(cfg), C.byref(w), kw["e"], 2, 8, kw["hidden"], kw["y"],
                                                    kw["ws"], kw["n"], None, None)
    assert call(**dict(ok, e=None)) == 1
    assert call(**dict(ok, y=P(264))) == 1
    assert call(**dict(ok, n=need - 1)) == 1 and "too small" in L.last_error()


def test_binding_declares_every_signature():
    # ctypes passes undeclared arguments as C ints: every entry point the
    # header declares must have its argument and result types set
    lib = L.lib()
    missing = [n for n in _declared() if getattr(lib, n).argtypes is None]
    assert not missing, missing
