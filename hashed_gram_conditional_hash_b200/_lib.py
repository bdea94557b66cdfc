"""ctypes binding of libengram (include/engram.h), argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors (device tensors where the header says DEVICE, numpy / sequences where
it says HOST), checks dtypes and contiguity, and passes raw pointers and the
current CUDA stream.  All computation happens in the CUDA kernels of
libengram.so; there is no fallback: if the library is missing the import of a
function raises.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libengram.so")

MAX_ORDERS = 8
ENGRAM_F32, ENGRAM_BF16 = 0, 1
STATUS_ID_RANGE, STATUS_ROW_RANGE, STATUS_TIMEOUT = 0x1, 0x2, 0x4
DEBUG_FORCE_TIMEOUT, DEBUG_FORCE_SIMT, DEBUG_FUSED_GATHER, DEBUG_TC_SINGLE_CTA, DEBUG_NO_PDL = 0x1, 0x2, 0x4, 0x8, 0x10
DEBUG_NO_OVERLAP = 0x20
DEBUG_TILE_MBLOCK_ORDER = 0x40
STATUS_NAMES = {0: "OK", 1: "ERR_INVALID_ARG", 2: "ERR_UNSUPPORTED", 3: "ERR_CUDA",
                4: "ERR_TIMEOUT", 5: "ERR_ID_RANGE"}


class EngramError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("%s: %s" % (STATUS_NAMES.get(code, code), msg))
        self.code = code


class EngramConfig(C.Structure):
    _fields_ = [("n_orders", C.c_int32), ("orders", C.c_int32 * MAX_ORDERS),
                ("heads_per_order", C.c_int32), ("row_dim", C.c_int32),
                ("hidden", C.c_int32), ("hc_mult", C.c_int32),
                ("conv_kernel", C.c_int32), ("dilation", C.c_int32),
                ("pad_id", C.c_int64), ("vocab", C.c_int64),
                ("rms_eps", C.c_float), ("gate_eps", C.c_float), ("dtype", C.c_int)]


class EngramWeights(C.Structure):
    _fields_ = [("table", C.c_void_p), ("total_rows", C.c_int64),
                ("row_offsets", C.c_void_p), ("primes", C.c_void_p),
                ("multipliers", C.c_void_p), ("lookup", C.c_void_p),
                ("raw_vocab", C.c_int64), ("w_value", C.c_void_p), ("w_key", C.c_void_p),
                ("norm_key", C.c_void_p), ("norm_query", C.c_void_p), ("conv_w", C.c_void_p)]


class EngramStageEvents(C.Structure):
    _fields_ = [("before_hash", C.c_void_p), ("before_projection", C.c_void_p),
                ("before_gate", C.c_void_p), ("before_conv", C.c_void_p),
                ("after_conv", C.c_void_p)]


class EngramState(C.Structure):
    _fields_ = [("id_ring", C.c_void_p), ("v_ring", C.c_void_p), ("g_ring", C.c_void_p),
                ("pos", C.c_void_p), ("ring_len", C.c_int32)]


_lib = None


def lib() -> C.CDLL:
    """Load libengram.so (built in-tree by build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libengram.so is missing at %s: run "
                               "hashed_gram_conditional_hash_b200/build.py (or "
                               "__graft_entry__.build()) first" % LIB_PATH)
        L = C.CDLL(LIB_PATH)
        P, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
        cfg = C.POINTER(EngramConfig)
        sig = {
            "engram_version": (i32, []),
            "engram_last_error": (sz, [C.c_char_p, sz]),
            "engram_read_status": (C.c_int, [P, P, P]),
            "engram_set_debug": (None, [C.c_uint32]),
            "engram_set_overlap_chunks": (None, [C.c_int32]),
            "engram_projection_engine": (i32, [cfg]),
            "engram_launch_count": (C.c_uint64, []),
            "engram_set_stage_events": (None, [C.POINTER(EngramStageEvents)]),
            "engram_compress_ids": (C.c_int, [P, i64, P, i64, P, P, P]),
            "engram_hash": (C.c_int, [cfg, P, i32, i32, P, P, P, P, P, P]),
            "engram_gather": (C.c_int, [cfg, P, i64, P, P, i64, P, P, P]),
            "engram_gate_fuse_workspace_size": (C.c_int, [cfg, i64, C.POINTER(sz)]),
            "engram_gate_fuse": (C.c_int, [cfg, P, P, P, P, P, P, i64, P, P, P, sz, P, P]),
            "engram_short_conv": (C.c_int, [cfg, P, i32, i32, P, P, P, P]),
            "engram_forward_workspace_size": (C.c_int, [cfg, i32, i32, C.POINTER(sz)]),
            "engram_state_init": (C.c_int, [cfg, C.POINTER(EngramState), i32, P]),
            "engram_forward": (C.c_int, [cfg, C.POINTER(EngramWeights), P, i32, i32, P, P,
                                         C.POINTER(EngramState), P, sz, P, P]),
            "engram_forward_no_alloc": (C.c_int, [cfg, C.POINTER(EngramWeights), P, i32, i32, P,
                                                  P, C.POINTER(EngramState), P, P]),
            "engram_gather_ids": (C.c_int, [cfg, C.POINTER(EngramWeights), P, i32, i32, P, P, P, P]),
            "engram_forward_gathered": (C.c_int, [cfg, C.POINTER(EngramWeights), P, i32, i32, P, P, P, sz,
                                                  P, P]),
            "engram_shard_rows": (i64, [i64, i32, i32]),
            "engram_shard_route_workspace_size": (sz, [cfg, i32, i32, i32]),
            "engram_shard_route": (C.c_int, [cfg, C.POINTER(EngramWeights), P, i32, i32, P, i32, P, P, P, P, sz,
                                             P, P]),
            "engram_shard_serve": (C.c_int, [cfg, P, i64, P, i64, P, P, P]),
            "engram_shard_place": (C.c_int, [cfg, P, P, i64, P, i64, P, P]),
            "engram_gather_ids_layers": (C.c_int, [cfg, C.POINTER(C.POINTER(EngramWeights)), i32, P, i32, i32,
                                                   P, C.POINTER(P), P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def last_error() -> str:
    buf = C.create_string_buffer(512)
    lib().engram_last_error(buf, 512)
    return buf.value.decode(errors="replace")


def _check(code: int):
    if code != 0:
        raise EngramError(code, last_error())


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libengram must be contiguous")
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _host_i64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int64))


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return ENGRAM_F32
    if dt == torch.bfloat16:
        return ENGRAM_BF16
    raise TypeError("libengram takes float32 or bfloat16 tensors, got %s" % dt)


def make_config(orders: Sequence[int], heads_per_order: int, row_dim: int, hidden: int,
                hc_mult: int, conv_kernel: int, dilation: int, pad_id: int, vocab: int,
                dtype: torch.dtype, rms_eps: float = 1e-6, gate_eps: float = 1e-6) -> EngramConfig:
    c = EngramConfig()
    c.n_orders = len(orders)
    for i, o in enumerate(orders):
        c.orders[i] = int(o)
    c.heads_per_order = heads_per_order
    c.row_dim = row_dim
    c.hidden = hidden
    c.hc_mult = hc_mult
    c.conv_kernel = conv_kernel
    c.dilation = dilation
    c.pad_id = pad_id
    c.vocab = vocab
    c.rms_eps = rms_eps
    c.gate_eps = gate_eps
    c.dtype = dtype_code(dtype)
    return c


# ---- entry points ---------------------------------------------------------

def engram_version() -> int:
    return lib().engram_version()


def engram_launch_count() -> int:
    return lib().engram_launch_count()


def engram_set_debug(flags: int) -> None:
    lib().engram_set_debug(flags)


def engram_set_overlap_chunks(chunks: int) -> None:
    """Sequence chunks of a prefill whose gate and conv overlap the next
    chunk's projection (<= 0: the default)."""
    lib().engram_set_overlap_chunks(chunks)


def engram_set_stage_events(events: Optional[dict]) -> None:
    """events: {stage name: torch.cuda.Event (already recorded once)} or None."""
    if events is None:
        lib().engram_set_stage_events(None)
        return
    ev = EngramStageEvents()
    for k, e in events.items():
        setattr(ev, k, e.cuda_event)
    lib().engram_set_stage_events(C.byref(ev))


ENGINE_SIMT, ENGINE_TCGEN05 = 0, 1


def engram_projection_engine(cfg: EngramConfig) -> int:
    return lib().engram_projection_engine(C.byref(cfg))


def engram_read_status(dev_status: torch.Tensor, stream=None) -> int:
    """Synchronises, returns the status bits and clears them (never raises on
    device bits; the C return code is folded into the bits)."""
    host = C.c_uint32(0)
    code = lib().engram_read_status(_ptr(dev_status), C.byref(host), _stream(stream))
    if code not in (0, 4, 5):
        _check(code)
    return host.value


def engram_compress_ids(raw: torch.Tensor, lookup: torch.Tensor, out: torch.Tensor,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    assert raw.dtype == lookup.dtype == out.dtype == torch.int64
    _check(lib().engram_compress_ids(_ptr(raw), raw.numel(), _ptr(lookup), lookup.numel(),
                                     _ptr(out), _ptr(dev_status), _stream(stream)))


def engram_hash(cfg: EngramConfig, ids: torch.Tensor, multipliers, primes, idx: torch.Tensor,
                history: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                stream=None) -> None:
    assert ids.dtype == idx.dtype == torch.int64 and ids.dim() == 2
    B, T = ids.shape
    m, p = _host_i64(multipliers), _host_i64(primes)
    _check(lib().engram_hash(C.byref(cfg), _ptr(ids), B, T, _ptr(history),
                             m.ctypes.data_as(C.c_void_p), p.ctypes.data_as(C.c_void_p),
                             _ptr(idx), _ptr(dev_status), _stream(stream)))


def engram_gather(cfg: EngramConfig, table: torch.Tensor, row_offsets, idx: torch.Tensor,
                  e: torch.Tensor, dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    nh = cfg.n_orders * cfg.heads_per_order
    M = idx.numel() // nh
    off = _host_i64(row_offsets)
    _check(lib().engram_gather(C.byref(cfg), _ptr(table), table.shape[0],
                               off.ctypes.data_as(C.c_void_p), _ptr(idx), M, _ptr(e),
                               _ptr(dev_status), _stream(stream)))


def engram_gate_fuse_workspace_size(cfg: EngramConfig, M: int) -> int:
    n = C.c_size_t(0)
    _check(lib().engram_gate_fuse_workspace_size(C.byref(cfg), M, C.byref(n)))
    return n.value


def engram_gate_fuse(cfg: EngramConfig, e, w_value, w_key, norm_key, norm_query, hidden,
                     u, gates=None, ws=None, dev_status=None, stream=None) -> None:
    M = e.shape[0]
    if ws is None:
        ws = torch.empty(engram_gate_fuse_workspace_size(cfg, M), dtype=torch.uint8,
                         device=e.device)
    _check(lib().engram_gate_fuse(C.byref(cfg), _ptr(e), _ptr(w_value), _ptr(w_key),
                                  _ptr(norm_key), _ptr(norm_query), _ptr(hidden), M, _ptr(u),
                                  _ptr(gates), _ptr(ws), ws.numel(), _ptr(dev_status),
                                  _stream(stream)))


def engram_short_conv(cfg: EngramConfig, u: torch.Tensor, conv_w: torch.Tensor, y: torch.Tensor,
                      conv_state: Optional[torch.Tensor] = None, stream=None) -> None:
    B, T = u.shape[0], u.shape[1]
    _check(lib().engram_short_conv(C.byref(cfg), _ptr(u), B, T, _ptr(conv_w), _ptr(conv_state),
                                   _ptr(y), _stream(stream)))


def engram_forward_workspace_size(cfg: EngramConfig, B: int, T: int) -> int:
    n = C.c_size_t(0)
    _check(lib().engram_forward_workspace_size(C.byref(cfg), B, T, C.byref(n)))
    return n.value


def engram_state_init(cfg: EngramConfig, state: EngramState, B: int, stream=None) -> None:
    _check(lib().engram_state_init(C.byref(cfg), C.byref(state), B, _stream(stream)))


def engram_forward(cfg: EngramConfig, weights: EngramWeights, ids: torch.Tensor,
                   hidden: torch.Tensor, y: torch.Tensor, ws: torch.Tensor,
                   state: Optional[EngramState] = None, dev_status: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    B, T = ids.shape
    _check(lib().engram_forward(C.byref(cfg), C.byref(weights), _ptr(ids), B, T, _ptr(hidden),
                                _ptr(y), C.byref(state) if state is not None else None, _ptr(ws),
                                ws.numel(), _ptr(dev_status), _stream(stream)))


def engram_gather_ids(cfg: EngramConfig, weights: EngramWeights, ids: torch.Tensor, e: torch.Tensor,
                      history: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    B, T = ids.shape
    _check(lib().engram_gather_ids(C.byref(cfg), C.byref(weights), _ptr(ids), B, T, _ptr(history), _ptr(e),
                                   _ptr(dev_status), _stream(stream)))


MAX_LAYERS = 4


def engram_gather_ids_layers(cfg: EngramConfig, weights: Sequence[EngramWeights], ids: torch.Tensor,
                             e: Sequence[torch.Tensor], history: Optional[torch.Tensor] = None,
                             dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    if len(weights) != len(e):
        raise ValueError("one output per layer")
    B, T = ids.shape
    n = len(weights)
    wp = (C.POINTER(EngramWeights) * n)(*[C.pointer(w) for w in weights])
    ep = (C.c_void_p * n)(*[_ptr(t).value for t in e])
    _check(lib().engram_gather_ids_layers(C.byref(cfg), wp, n, _ptr(ids), B, T, _ptr(history), ep,
                                          _ptr(dev_status), _stream(stream)))


MAX_SHARDS = 64


def engram_shard_rows(total_rows: int, n_shards: int, shard: int) -> int:
    """Rows held by shard ``shard`` (stacked-table rows shard, shard + n_shards, ...)."""
    n = lib().engram_shard_rows(total_rows, n_shards, shard)
    if n < 0:
        raise ValueError("shard %d of %d out of range" % (shard, n_shards))
    return n


def engram_shard_route_workspace_size(cfg: EngramConfig, B: int, T: int, n_shards: int) -> int:
    return lib().engram_shard_route_workspace_size(C.byref(cfg), B, T, n_shards)


def engram_shard_route(cfg: EngramConfig, weights: EngramWeights, ids: torch.Tensor, n_shards: int,
                       counts: torch.Tensor, req_rows: torch.Tensor, req_pos: torch.Tensor, ws: torch.Tensor,
                       history: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                       stream=None) -> None:
    B, T = ids.shape
    _check(lib().engram_shard_route(C.byref(cfg), C.byref(weights), _ptr(ids), B, T, _ptr(history), n_shards,
                                    _ptr(counts), _ptr(req_rows), _ptr(req_pos), _ptr(ws), ws.numel(),
                                    _ptr(dev_status), _stream(stream)))


def engram_shard_serve(cfg: EngramConfig, shard: torch.Tensor, req_rows: torch.Tensor, out: torch.Tensor,
                       dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().engram_shard_serve(C.byref(cfg), _ptr(shard), shard.shape[0], _ptr(req_rows), req_rows.numel(),
                                    _ptr(out), _ptr(dev_status), _stream(stream)))


def engram_shard_place(cfg: EngramConfig, got: torch.Tensor, req_pos: torch.Tensor, e: torch.Tensor,
                       n_e: int, dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().engram_shard_place(C.byref(cfg), _ptr(got), _ptr(req_pos), req_pos.numel(), _ptr(e), n_e,
                                    _ptr(dev_status), _stream(stream)))


def engram_forward_gathered(cfg: EngramConfig, weights: EngramWeights, e: torch.Tensor, B: int, T: int,
                            hidden: torch.Tensor, y: torch.Tensor, ws: torch.Tensor,
                            dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    _check(lib().engram_forward_gathered(C.byref(cfg), C.byref(weights), _ptr(e), B, T, _ptr(hidden), _ptr(y),
                                         _ptr(ws), ws.numel(), _ptr(dev_status), _stream(stream)))


NO_ALLOC_SCRATCH_BYTES = 32 << 20


def engram_forward_no_alloc(cfg: EngramConfig, weights: EngramWeights, ids: torch.Tensor,
                            hidden: torch.Tensor, y: torch.Tensor,
                            state: Optional[EngramState] = None,
                            dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """engram_forward in the library's static device scratch (no workspace
    argument; for callers that cannot allocate device memory)."""
    B, T = ids.shape
    _check(lib().engram_forward_no_alloc(C.byref(cfg), C.byref(weights), _ptr(ids), B, T,
                                         _ptr(hidden), _ptr(y),
                                         C.byref(state) if state is not None else None,
                                         _ptr(dev_status), _stream(stream)))
