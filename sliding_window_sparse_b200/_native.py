"""ctypes view of ``libswa.so`` (the C ABI of include/swa.h).

Loading fails loudly when the library is missing: there is no other
implementation behind these names.
"""

from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libswa.so")

_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_p = ctypes.c_void_p
_sz = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/swa.h
SIGNATURES = {
    "swa_status_string": (ctypes.c_char_p, [_i]),
    "swa_version": (_i, []),
    "swa_block_meta": (_i, [_i, _i, _i64, _i64, _p, _i64, _i, _i, _p, _p, _p]),
    "swa_attn_fwd": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i64, _i, _i64, _f, _p]),
    "swa_attn_chunk_ring": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i64, _i, _i64, _f,
                                 _i, _p]),
    "swa_attn_fwd_sink": (_i, [_p, _p, _p, _p, _p, _i, _i, _i, _i64, _i, _i64, _i, _f, _p]),
    "swa_attn_varlen": (_i, [_p, _p, _p, _p, _p, _p, _i, _i64, _i64, _i, _i, _i, _i64, _i, _f,
                             _p]),
    "swa_attn_decode_ring_sink": (_i, [_p, _p, _p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i, _i64,
                                       _f, _p, _sz, _p]),
    "swa_attn_bwd_workspace_bytes": (_sz, [_i, _i, _i64]),
    "swa_attn_bwd": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i64, _i, _i64, _f, _p,
                          _sz, _p]),
    "swa_attn_bwd_sink": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i64, _i, _i64, _i,
                               _f, _p, _sz, _p]),
    "swa_attn_varlen_bwd_workspace_bytes": (_sz, [_i, _i64]),
    "swa_attn_varlen_bwd": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i64, _i64, _i, _i,
                                 _i, _i64, _i, _f, _p, _sz, _p]),
    "swa_attn_chunk_ring_sink": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _p, _p, _p, _i, _i, _i, _i64,
                                      _i, _i64, _f, _i, _p]),
    "swa_attn_chunk_ring_ragged": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i64, _i,
                                        _i64, _f, _i, _p]),
    "swa_chunk_split_workspace_bytes": (_sz, [_i, _i, _i, _i64, _i, _i64]),
    "swa_attn_chunk_ring_split": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _p, _p, _p, _p, _i, _i, _i,
                                       _i64, _i, _i64, _f, _i, _p, _sz, _p]),
    "swa_ring_write": (_i, [_p, _p, _p, _p, _p, _i, _i, _i64, _i, _i64, _p]),
    "swa_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i64]),
    "swa_attn_decode_ring": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i64, _f, _p, _sz, _p]),
    "swa_ring_slot_positions": (_i, [_i, _p, _i64, _p, _p]),
    "swa_attn_decode_ring_static": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i64, _f, _p]),
    "swa_selftest_wait": (_i, [_i64, _i, _p, _p]),
    "swa_get_device_status": (_i, [_p]),
}

_lock = threading.Lock()
_lib = None


class SwaError(RuntimeError):
    """A libswa call returned a non-zero status."""

    def __init__(self, fn: str, status: int, name: str):
        super().__init__(f"{fn} failed: {name} ({status})")
        self.status = status
        self.fn = fn


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it was never built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m sliding_window_sparse_b200.build` (needs nvcc)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(handle, name)
                fn.restype = res
                fn.argtypes = args
            _lib = handle
    return _lib


def status_name(status: int) -> str:
    return lib().swa_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != 0:
        raise SwaError(fn, status, status_name(status))
