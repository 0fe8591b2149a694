"""fp64 CPU oracle for causal sliding-window attention -- test infrastructure.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package.  The library in
``sliding_window_sparse_b200`` never imports it, and the two share no code:
the oracle is ``swa_oracle.c`` (plain C, fp64 loops), compiled here with gcc
into ``liboracle.so`` and called through ctypes.

Every entry point takes the raw bfloat16 bit patterns (``uint16`` numpy
arrays, C order) produced by :mod:`swa_inputs` and returns float64 results.

Functions and the passages they follow (page title, section):

* :func:`count_pairs`     -- M003 note section 03 (allowed pairs; 21 vs 36).
* :func:`swa_forward`     -- M003 note section 03; Chapter 10 section 10.1.
* :func:`dense_masked`    -- M003 note section 07 (dense table + mask baseline),
                             Chapter 10 section 10.1 (diff convention).
* :func:`ring_positions`  -- "Dense attention vs sparse SWA" blog section 3.2
                             (circular cache write procedure).
* :func:`swa_chunk`       -- Chapter 10 section 10.2 (chunk union W + T_q - 1),
                             M003 note section 06.
* :func:`ring_update`     -- Chapter 10 section 10.2; blog section 3.2.
* :func:`swa_decode`      -- blog section 3.2; taxonomy page section 1.
* :func:`tile_classes`    -- M003 note section 04 (skip / full / partial tiles).
* :func:`count_pairs_sink` -- taxonomy page section 3.2 (StreamingLLM: first
                             tokens plus the recent W), by enumeration.
* :func:`swa_varlen`      -- blog section 5.2 tip 4 (packed batches, windows per
                             sequence via cu_seqlens), with optional sinks.
* :func:`swa_decode_sink` -- taxonomy page section 3.2 on top of the ring decode.
* :func:`swa_chunk_sink`  -- taxonomy page section 3.2 on top of the chunked prefill.
* :func:`swa_backward`    -- M003 note sections 07-08 (Q/K/V gradients under the
                             same mask); :func:`swa_forward_f64` is the forward
                             on fp64 inputs that its finite differences use.
* :func:`swa_varlen_backward` -- the same gradients for packed sequences with
                             optional sinks (blog section 5.2 tip 4, taxonomy
                             page section 3.2); :func:`swa_varlen_f64` is its
                             fp64 forward.

All of them are pinned by ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dbl = ctypes.c_double
_ptr = ctypes.c_void_p


def build(force: bool = False) -> str:
    """Compile ``swa_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
               "-std=c11", "-Wall", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = _configure(ctypes.CDLL(_LIB))
            _lib = lib
    return _lib


def _configure(lib):
    """Declare the C signatures on a loaded build of swa_oracle.c."""
    lib.orc_num_threads.restype = _int
    lib.orc_count_pairs.restype = _i64
    lib.orc_count_pairs.argtypes = [_i64, _i64]
    lib.orc_swa_forward.restype = _i64
    lib.orc_swa_forward.argtypes = [_ptr, _ptr, _ptr, _int, _int, _int, _i64, _int, _i64,
                                    _dbl, _ptr, _ptr, _i64, _ptr, _ptr]
    lib.orc_dense_masked.restype = _int
    lib.orc_dense_masked.argtypes = [_ptr, _ptr, _ptr, _int, _int, _int, _i64, _int, _i64,
                                     _dbl, _ptr]
    lib.orc_ring_positions.restype = None
    lib.orc_ring_positions.argtypes = [_i64, _i64, _ptr]
    lib.orc_swa_chunk.restype = _i64
    lib.orc_swa_chunk.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _int, _int, _int,
                                  _i64, _int, _i64, _dbl, _ptr, _i64, _ptr, _ptr]
    lib.orc_ring_update.restype = None
    lib.orc_ring_update.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _int, _int, _i64, _int,
                                    _i64]
    lib.orc_swa_decode.restype = _i64
    lib.orc_swa_decode.argtypes = [_ptr, _ptr, _ptr, _ptr, _int, _int, _int, _int, _i64,
                                   _dbl, _ptr, _ptr]
    lib.orc_count_pairs_sink.restype = _i64
    lib.orc_count_pairs_sink.argtypes = [_i64, _i64, _i64]
    lib.orc_swa_varlen.restype = _i64
    lib.orc_swa_varlen.argtypes = [_ptr, _ptr, _ptr, _ptr, _int, _int, _int, _int, _i64, _i64,
                                   _dbl, _ptr, _i64, _ptr, _ptr]
    lib.orc_swa_decode_sink.restype = _i64
    lib.orc_swa_decode_sink.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _int, _int, _int,
                                        _int, _i64, _i64, _dbl, _ptr, _ptr]
    lib.orc_swa_chunk_sink.restype = _i64
    lib.orc_swa_chunk_sink.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _i64, _ptr, _int,
                                       _int, _int, _i64, _int, _i64, _dbl, _ptr, _i64, _ptr, _ptr]
    lib.orc_swa_forward_f64.restype = _i64
    lib.orc_swa_forward_f64.argtypes = [_ptr, _ptr, _ptr, _int, _int, _int, _i64, _int, _i64,
                                        _dbl, _ptr]
    lib.orc_swa_backward.restype = _i64
    lib.orc_swa_backward.argtypes = [_ptr, _ptr, _ptr, _ptr, _int, _int, _int, _i64, _int, _i64,
                                     _dbl, _ptr, _ptr, _ptr]
    lib.orc_swa_varlen_f64.restype = _i64
    lib.orc_swa_varlen_f64.argtypes = [_ptr, _ptr, _ptr, _ptr, _int, _int, _int, _int, _i64,
                                       _i64, _dbl, _ptr]
    lib.orc_swa_varlen_backward.restype = _i64
    lib.orc_swa_varlen_backward.argtypes = [_ptr, _ptr, _ptr, _ptr, _ptr, _int, _int, _int, _int,
                                            _i64, _i64, _dbl, _ptr, _ptr, _ptr]
    lib.orc_tile_classes.restype = _int
    lib.orc_tile_classes.argtypes = [_int, _int, _i64, _i64, _ptr, _i64, _int, _int, _ptr,
                                     _ptr]
    return lib


class use_library:
    """Context manager (tests only): route every oracle call to another build of
    swa_oracle.c, e.g. a copy with a planted mistake, then restore."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        _load()
        with _lock:
            self.saved = _lib
            _lib = _configure(ctypes.CDLL(self.path))
        return self

    def __exit__(self, *exc):
        global _lib
        with _lock:
            _lib = self.saved
        return False


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bfloat16 bit patterns (numpy uint16)")
    return a


def _rows(rows):
    if rows is None:
        return None
    r = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    return r


def num_threads() -> int:
    """OpenMP threads the oracle uses."""
    return int(_load().orc_num_threads())


def count_pairs(N: int, W: int) -> int:
    """Allowed (query, key) pairs among N positions, by enumeration."""
    return int(_load().orc_count_pairs(N, W))


def swa_forward(q, k, v, W: int, scale: float, rows=None, q_pos0=None, with_lse=False):
    """Sliding-window attention over a linear layout.

    q: [B,H,N,d], k/v: [B,Hkv,N,d] bf16 bits.  ``rows``: optional (n,3) int64
    array of (b, h, i); the result is then [n, d] instead of [B,H,N,d].
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    r = _rows(rows)
    n = r.shape[0] if r is not None else B * H * N
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64) if with_lse else None
    qp = None if q_pos0 is None else np.ascontiguousarray(q_pos0, dtype=np.int64)
    bad = _load().orc_swa_forward(_p(q), _p(k), _p(v), B, H, Hkv, N, d, W, scale, _p(qp),
                                  _p(r), n, _p(out), _p(lse))
    if bad:
        raise ValueError(f"{bad} query rows have no legal key")
    if r is None:
        out = out.reshape(B, H, N, d)
        if lse is not None:
            lse = lse.reshape(B, H, N)
    return (out, lse) if with_lse else out


def count_pairs_sink(N: int, W: int, n_sink: int) -> int:
    """Visible pairs among N positions with the window plus the first n_sink keys."""
    return int(_load().orc_count_pairs_sink(N, W, n_sink))


def swa_varlen(q, k, v, cu_seqlens, W: int, scale: float, n_sink: int = 0, rows=None,
               with_lse=False):
    """Packed variable-length attention, per-sequence windows (and sinks).

    q: [total,H,d], k/v: [total,Hkv,d] bf16 bits; cu_seqlens: [n_seq+1] int64 from 0.
    ``rows``: optional (n,2) int64 array of (token, h); the result is then [n, d]
    instead of [total,H,d] (lse [n] instead of [total,H]).
    """
    q, k, v = _u16(q), _u16(k), _u16(v)
    total, H, d = q.shape
    Hkv = k.shape[1]
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64).reshape(-1)
    if cu[-1] != total:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 2)
    n = r.shape[0] if r is not None else total * H
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64) if with_lse else None
    bad = _load().orc_swa_varlen(_p(q), _p(k), _p(v), _p(cu), cu.shape[0] - 1, H, Hkv, d, W,
                                 n_sink, scale, _p(r), n, _p(out), _p(lse))
    if bad < 0:
        raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
    if bad:
        raise ValueError(f"{bad} query rows have no legal key")
    if r is None:
        out = out.reshape(total, H, d)
        if lse is not None:
            lse = lse.reshape(total, H)
    return (out, lse) if with_lse else out


def _f64(a):
    """bf16 bit patterns (uint16) -> their exact values; float arrays -> float64."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ascontiguousarray(a, dtype=np.float64)


def swa_forward_f64(q, k, v, W: int, scale: float):
    """swa_forward on fp64 inputs (the function the gradient pins differentiate)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    out = np.empty((B, H, N, d), dtype=np.float64)
    if _load().orc_swa_forward_f64(_p(q), _p(k), _p(v), B, H, k.shape[1], N, d, W, scale,
                                   _p(out)):
        raise ValueError("query rows without a legal key")
    return out


def swa_backward(q, k, v, dout, W: int, scale: float):
    """Gradients (dq, dk, dv) of sum(out * dout) for the linear prefill, in fp64.

    q, dout: [B,H,N,d]; k, v: [B,Hkv,N,d]; bf16 bits or float arrays.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    dq = np.empty((B, H, N, d), dtype=np.float64)
    dk = np.empty((B, Hkv, N, d), dtype=np.float64)
    dv = np.empty((B, Hkv, N, d), dtype=np.float64)
    if _load().orc_swa_backward(_p(q), _p(k), _p(v), _p(dout), B, H, Hkv, N, d, W, scale,
                                _p(dq), _p(dk), _p(dv)):
        raise ValueError("query rows without a legal key")
    return dq, dk, dv


def _cu(cu_seqlens, total):
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64).reshape(-1)
    if cu[-1] != total:
        raise ValueError("cu_seqlens[-1] must equal the packed token count")
    return cu


def swa_varlen_f64(q, k, v, cu_seqlens, W: int, scale: float, n_sink: int = 0):
    """swa_varlen on fp64 inputs (the function the varlen gradient pins differentiate).

    q: [total,H,d], k/v: [total,Hkv,d]; bf16 bits or float arrays.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    total, H, d = q.shape
    cu = _cu(cu_seqlens, total)
    out = np.empty((total, H, d), dtype=np.float64)
    bad = _load().orc_swa_varlen_f64(_p(q), _p(k), _p(v), _p(cu), cu.shape[0] - 1, H,
                                     k.shape[1], d, W, n_sink, scale, _p(out))
    if bad:
        raise ValueError("malformed cu_seqlens" if bad < 0 else "query rows without a legal key")
    return out


def swa_varlen_backward(q, k, v, dout, cu_seqlens, W: int, scale: float, n_sink: int = 0):
    """Gradients (dq, dk, dv) of sum(out * dout) for the packed varlen prefill
    (per-sequence windows, optional sinks), in fp64.

    q, dout: [total,H,d]; k, v: [total,Hkv,d]; bf16 bits or float arrays.
    """
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    total, H, d = q.shape
    Hkv = k.shape[1]
    cu = _cu(cu_seqlens, total)
    dq = np.empty((total, H, d), dtype=np.float64)
    dk = np.empty((total, Hkv, d), dtype=np.float64)
    dv = np.empty((total, Hkv, d), dtype=np.float64)
    bad = _load().orc_swa_varlen_backward(_p(q), _p(k), _p(v), _p(dout), _p(cu),
                                          cu.shape[0] - 1, H, Hkv, d, W, n_sink, scale,
                                          _p(dq), _p(dk), _p(dv))
    if bad:
        raise ValueError("malformed cu_seqlens" if bad < 0 else "query rows without a legal key")
    return dq, dk, dv


def dense_masked(q, k, v, W: int, scale: float):
    """Dense score table + window mask + row softmax (positions 0..N-1)."""
    q, k, v = _u16(q), _u16(k), _u16(v)
    B, H, N, d = q.shape
    out = np.empty((B, H, N, d), dtype=np.float64)
    if _load().orc_dense_masked(_p(q), _p(k), _p(v), B, H, k.shape[1], N, d, W, scale, _p(out)):
        raise MemoryError("dense_masked: allocation failed")
    return out


def ring_positions(n_written: int, W: int) -> np.ndarray:
    """Logical position held by each of the W slots after writing 0..n_written-1 (-1 = empty)."""
    out = np.empty(W, dtype=np.int64)
    _load().orc_ring_positions(n_written, W, _p(out))
    return out


def swa_chunk(q, k_new, v_new, ring_k, ring_v, q_start, W: int, scale: float, rows=None,
              with_lse=False):
    """Chunked prefill: queries at q_start[b]+t over ring (positions < q_start) + chunk."""
    q, k_new, v_new = _u16(q), _u16(k_new), _u16(v_new)
    ring_k, ring_v = _u16(ring_k), _u16(ring_v)
    B, H, Tq, d = q.shape
    Hkv = k_new.shape[1]
    qs = np.ascontiguousarray(q_start, dtype=np.int64).reshape(B)
    r = _rows(rows)
    n = r.shape[0] if r is not None else B * H * Tq
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64) if with_lse else None
    bad = _load().orc_swa_chunk(_p(q), _p(k_new), _p(v_new), _p(ring_k), _p(ring_v), _p(qs),
                                B, H, Hkv, Tq, d, W, scale, _p(r), n, _p(out), _p(lse))
    if bad:
        raise ValueError(f"{bad} query rows have a missing or no legal key")
    if r is None:
        out = out.reshape(B, H, Tq, d)
        if lse is not None:
            lse = lse.reshape(B, H, Tq)
    return (out, lse) if with_lse else out


def swa_chunk_sink(q, k_new, v_new, ring_k, ring_v, sink_k, sink_v, q_start, W: int,
                   scale: float, rows=None, with_lse=False):
    """swa_chunk with sink rows [B,Hkv,S,d] holding positions 0..S-1."""
    q, k_new, v_new = _u16(q), _u16(k_new), _u16(v_new)
    ring_k, ring_v, sink_k, sink_v = _u16(ring_k), _u16(ring_v), _u16(sink_k), _u16(sink_v)
    B, H, Tq, d = q.shape
    Hkv, S = k_new.shape[1], sink_k.shape[2]
    qs = np.ascontiguousarray(q_start, dtype=np.int64).reshape(B)
    r = _rows(rows)
    n = r.shape[0] if r is not None else B * H * Tq
    out = np.empty((n, d), dtype=np.float64)
    lse = np.empty(n, dtype=np.float64) if with_lse else None
    bad = _load().orc_swa_chunk_sink(_p(q), _p(k_new), _p(v_new), _p(ring_k), _p(ring_v),
                                     _p(sink_k), _p(sink_v), S, _p(qs), B, H, Hkv, Tq, d, W,
                                     scale, _p(r), n, _p(out), _p(lse))
    if bad:
        raise ValueError(f"{bad} query rows have a missing or no legal key")
    if r is None:
        out = out.reshape(B, H, Tq, d)
        if lse is not None:
            lse = lse.reshape(B, H, Tq)
    return (out, lse) if with_lse else out


def ring_update(k_new, v_new, ring_k, ring_v, q_start, W: int):
    """Return copies of (ring_k, ring_v) after writing the chunk's positions."""
    k_new, v_new = _u16(k_new), _u16(v_new)
    rk = _u16(ring_k).copy()
    rv = _u16(ring_v).copy()
    B, Hkv, Tq, d = k_new.shape
    qs = np.ascontiguousarray(q_start, dtype=np.int64).reshape(B)
    _load().orc_ring_update(_p(k_new), _p(v_new), _p(rk), _p(rv), _p(qs), B, Hkv, Tq, d, W)
    return rk, rv


def swa_decode(q, ring_k, ring_v, pos, W: int, scale: float, with_lse=False):
    """One query per sequence at position pos[b]; the ring already holds it."""
    q, ring_k, ring_v = _u16(q), _u16(ring_k), _u16(ring_v)
    B, H, d = q.shape
    Hkv = ring_k.shape[1]
    p = np.ascontiguousarray(pos, dtype=np.int64).reshape(B)
    out = np.empty((B, H, d), dtype=np.float64)
    lse = np.empty((B, H), dtype=np.float64) if with_lse else None
    bad = _load().orc_swa_decode(_p(q), _p(ring_k), _p(ring_v), _p(p), B, H, Hkv, d, W, scale,
                                 _p(out), _p(lse))
    if bad:
        raise ValueError(f"{bad} decode rows have a missing or no legal key")
    return (out, lse) if with_lse else out


def swa_decode_sink(q, ring_k, ring_v, sink_k, sink_v, pos, W: int, scale: float,
                    with_lse=False):
    """Decode over a ring plus sink rows [B,Hkv,S,d] holding positions 0..S-1."""
    q, ring_k, ring_v = _u16(q), _u16(ring_k), _u16(ring_v)
    sink_k, sink_v = _u16(sink_k), _u16(sink_v)
    B, H, d = q.shape
    Hkv, S = sink_k.shape[1], sink_k.shape[2]
    p = np.ascontiguousarray(pos, dtype=np.int64).reshape(B)
    out = np.empty((B, H, d), dtype=np.float64)
    lse = np.empty((B, H), dtype=np.float64) if with_lse else None
    bad = _load().orc_swa_decode_sink(_p(q), _p(ring_k), _p(ring_v), _p(sink_k), _p(sink_v),
                                      _p(p), B, H, Hkv, d, W, S, scale, _p(out), _p(lse))
    if bad:
        raise ValueError(f"{bad} decode rows have a missing or no legal key")
    return (out, lse) if with_lse else out


def tile_classes(mode: int, B: int, n_q: int, n_k: int, W: int, tile_q: int, tile_k: int,
                 q_pos0=None):
    """Brute-force tile classes (0 skip, 1 full, 2 partial) and per-row-tile ranges.

    Returns (classes int8 [B,nqt,nkt], ranges int32 [B,nqt,4]) with ranges =
    (live tiles, full tiles, first live tile, last live tile).
    """
    nqt = (n_q + tile_q - 1) // tile_q
    if mode == 1:
        nkt = (W + tile_k - 1) // tile_k + (n_q + tile_k - 1) // tile_k
    else:
        nkt = (n_k + tile_k - 1) // tile_k
    cls = np.empty((B, nqt, nkt), dtype=np.int8)
    rng = np.empty((B, nqt, 4), dtype=np.int32)
    qp = None if q_pos0 is None else np.ascontiguousarray(q_pos0, dtype=np.int64).reshape(B)
    _load().orc_tile_classes(mode, B, n_q, n_k, _p(qp), W, tile_q, tile_k, _p(cls), _p(rng))
    return cls, rng
