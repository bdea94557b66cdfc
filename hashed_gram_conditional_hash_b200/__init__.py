"""libengram: the Engram conditional-memory forward pass as hand-written
sm_100a CUDA behind a C ABI (include/engram.h), with a thin ctypes binding."""
from . import _lib
from ._lib import (EngramError, engram_compress_ids, engram_forward,
                   engram_forward_workspace_size, engram_gate_fuse,
                   engram_gate_fuse_workspace_size, engram_gather, engram_hash,
                   engram_projection_engine,
                   engram_read_status, engram_set_debug, engram_short_conv,
                   engram_state_init, engram_version)
from .layer import EngramLayer, StreamState
from .sharded import ShardedGather

__all__ = [
    "EngramError", "EngramLayer", "ShardedGather", "StreamState", "engram_compress_ids", "engram_forward",
    "engram_forward_workspace_size", "engram_gate_fuse", "engram_gate_fuse_workspace_size",
    "engram_gather", "engram_hash", "engram_projection_engine", "engram_read_status", "engram_set_debug",
    "engram_short_conv", "engram_state_init", "engram_version",
]
