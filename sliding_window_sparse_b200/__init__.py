"""Causal sliding-window attention for NVIDIA B200 (sm_100a).

A query at logical position i reads the keys at positions
max(0, i - W + 1) .. i (the window includes the query's own position), and
the softmax is taken over those pairs only.  Every step runs in the CUDA
kernels of ``libswa.so`` behind the C ABI of ``include/swa.h``; this module
only marshals torch tensors (device memory, current stream) into those calls.
The function names match the C entry points.  One addition sits above them:
``swa_attn_fwd_seq_parallel`` (module ``seq_parallel``) splits a sequence
along its length across ``torch.distributed`` ranks; it exchanges the W - 1
key/value rows before each shard and then calls ``swa_ring_write`` and
``swa_attn_chunk_ring``.

Layouts (row-major bf16): queries ``[B, H, rows, d]``, keys/values
``[B, Hkv, rows, d]``, ring caches ``[B, Hkv, W, d]``; query head h reads
key/value head ``h // (H // Hkv)``.
"""

from __future__ import annotations

import math

import torch

from ._native import SwaError, check, lib, status_name  # noqa: F401

__all__ = [
    "SwaError",
    "lib",
    "swa_block_meta",
    "swa_attn_fwd",
    "swa_attn_fwd_sink",
    "swa_attn_bwd",
    "swa_attn_varlen_bwd",
    "swa_attn_varlen",
    "swa_attn_chunk_ring",
    "swa_attn_chunk_ring_ragged",
    "swa_attn_chunk_ring_sink",
    "swa_attn_chunk_ring_split",
    "swa_chunk_split_workspace_bytes",
    "swa_ring_write",
    "swa_decode_workspace_bytes",
    "swa_attn_decode_ring",
    "swa_attn_decode_ring_sink",
    "swa_attn_decode_ring_static",
    "swa_ring_slot_positions",
    "swa_selftest_wait",
    "swa_get_device_status",
    "swa_version",
    "swa_attn_fwd_seq_parallel",
]


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(device=None):
    return torch.cuda.current_stream(device).cuda_stream


def _need(t, name, dtype=torch.bfloat16, dims=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dims, got {t.dim()}")


def swa_version() -> int:
    return int(lib().swa_version())


def swa_block_meta(key_mode: int, n_q: int, n_k: int, W: int, tile_q: int, tile_k: int,
                   q_pos0: torch.Tensor | None = None, B: int | None = None,
                   classes: torch.Tensor | None = None, ranges: torch.Tensor | None = None,
                   device=None):
    """Tile classes (int8 [B,nqt,nkt]: 0 skip, 1 full, 2 partial) and ranges (int32 [B,nqt,4])."""
    if q_pos0 is not None:
        _need(q_pos0, "q_pos0", torch.int64, 1)
        B = q_pos0.numel()
        device = q_pos0.device
    if B is None:
        raise ValueError("B is required when q_pos0 is None")
    device = torch.device("cuda") if device is None else torch.device(device)
    nqt = (n_q + tile_q - 1) // tile_q
    nkt = ((n_k + tile_k - 1) // tile_k if key_mode == 0
           else (W + tile_k - 1) // tile_k + (n_q + tile_k - 1) // tile_k)
    if classes is None:
        classes = torch.empty((B, nqt, nkt), dtype=torch.int8, device=device)
    if ranges is None:
        ranges = torch.empty((B, nqt, 4), dtype=torch.int32, device=device)
    check("swa_block_meta", lib().swa_block_meta(key_mode, B, n_q, n_k, _ptr(q_pos0), W, tile_q,
                                                 tile_k, _ptr(classes), _ptr(ranges),
                                                 _stream(device)))
    return classes, ranges


def swa_attn_fwd(q, k, v, W: int, scale: float | None = None, out=None, lse=None,
                 return_lse: bool = False, n_sink: int = 0):
    """Prefill forward: q [B,H,N,d], k/v [B,Hkv,N,d] -> out [B,H,N,d] (and lse [B,H,N]).

    n_sink > 0 keeps keys 0..n_sink-1 visible to every later query (swa_attn_fwd_sink).
    """
    _need(q, "q", dims=4)
    _need(k, "k", dims=4)
    _need(v, "v", dims=4)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, N, d) or tuple(v.shape) != (B, Hkv, N, d):
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", dims=4)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
    if n_sink:
        check("swa_attn_fwd_sink",
              lib().swa_attn_fwd_sink(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Hkv,
                                      N, d, W, n_sink, scale, _stream(q.device)))
    else:
        check("swa_attn_fwd", lib().swa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                                 B, H, Hkv, N, d, W, scale, _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_attn_bwd(q, k, v, out, dout, lse, W: int, scale: float | None = None, dq=None, dk=None,
                 dv=None, workspace=None, n_sink: int = 0):
    """Gradients of swa_attn_fwd: returns (dq [B,H,N,d], dk, dv [B,Hkv,N,d]).

    out and lse are the forward's output and natural-log LSE; dout is the incoming gradient.
    n_sink > 0: gradients of swa_attn_fwd_sink with the same sinks (swa_attn_bwd_sink).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, dims=4)
    _need(lse, "lse", torch.float32, 3)
    B, H, N, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (B, Hkv, N, d) or tuple(v.shape) != (B, Hkv, N, d):
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    if tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("out and dout must match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = int(lib().swa_attn_bwd_workspace_bytes(B, H, N))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if n_sink:
        check("swa_attn_bwd_sink",
              lib().swa_attn_bwd_sink(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, N, d, W, n_sink,
                                      scale, _ptr(workspace), ws_bytes, _stream(q.device)))
    else:
        check("swa_attn_bwd",
              lib().swa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
                                 _ptr(dq), _ptr(dk), _ptr(dv), B, H, Hkv, N, d, W, scale,
                                 _ptr(workspace), ws_bytes, _stream(q.device)))
    return dq, dk, dv


def swa_attn_varlen_bwd(q, k, v, cu_seqlens, max_seqlen: int, out, dout, lse, W: int,
                        scale: float | None = None, n_sink: int = 0, dq=None, dk=None, dv=None,
                        workspace=None):
    """Gradients of swa_attn_varlen: returns (dq [total,H,d], dk, dv [total,Hkv,d]).

    out and lse ([H, total]) are the forward's; dout is the incoming gradient.  Rows of
    tokens outside every sequence keep what dq / dk / dv held (zeros when allocated here).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _need(t, n, dims=3)
    _need(cu_seqlens, "cu_seqlens", torch.int64, 1)
    _need(lse, "lse", torch.float32, 2)
    total, H, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (total, Hkv, d) or tuple(v.shape) != (total, Hkv, d):
        raise ValueError("k and v must be [total, Hkv, d] matching q")
    if tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape):
        raise ValueError("out and dout must match q")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.zeros_like(q) if dq is None else dq
    dk = torch.zeros_like(k) if dk is None else dk
    dv = torch.zeros_like(v) if dv is None else dv
    need = int(lib().swa_attn_varlen_bwd_workspace_bytes(H, total))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check("swa_attn_varlen_bwd",
          lib().swa_attn_varlen_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(out),
                                    _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                                    cu_seqlens.shape[0] - 1, total, max_seqlen, H, Hkv, d, W,
                                    n_sink, scale, _ptr(workspace),
                                    workspace.numel() * workspace.element_size(),
                                    _stream(q.device)))
    return dq, dk, dv


def swa_attn_varlen(q, k, v, cu_seqlens, max_seqlen: int, W: int, scale: float | None = None,
                    n_sink: int = 0, out=None, lse=None, return_lse: bool = False):
    """Packed prefill: q [total,H,d], k/v [total,Hkv,d], cu_seqlens int64 [n_seq+1] (device).

    Each sequence has its own positions and window; returns out [total,H,d] (and
    lse [H,total]).  Rows of tokens outside every sequence keep what `out` held.
    """
    _need(q, "q", dims=3)
    _need(k, "k", dims=3)
    _need(v, "v", dims=3)
    _need(cu_seqlens, "cu_seqlens", torch.int64, 1)
    total, H, d = q.shape
    Hkv = k.shape[1]
    if tuple(k.shape) != (total, Hkv, d) or tuple(v.shape) != (total, Hkv, d):
        raise ValueError("k and v must be [total, Hkv, d] matching q")
    n_seq = cu_seqlens.shape[0] - 1
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.zeros_like(q)
    _need(out, "out", dims=3)
    if return_lse and lse is None:
        lse = torch.zeros((H, total), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
    check("swa_attn_varlen",
          lib().swa_attn_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(out), _ptr(lse),
                                n_seq, total, max_seqlen, H, Hkv, d, W, n_sink, scale,
                                _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_attn_chunk_ring(q, k_new, v_new, k_ring, v_ring, q_start, scale: float | None = None,
                        update_ring: bool = False, out=None, lse=None, return_lse: bool = False,
                        k_sink=None, v_sink=None):
    """Chunked prefill on a ring cache: q [B,H,Tq,d], chunk k/v [B,Hkv,Tq,d], ring [B,Hkv,W,d].

    With k_sink / v_sink [B,Hkv,S,d] (positions 0..S-1) the sinks before each window
    are attended too (swa_attn_chunk_ring_sink).
    """
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_ring, "k_ring"),
                 (v_ring, "v_ring")):
        _need(t, n, dims=4)
    _need(q_start, "q_start", torch.int64, 1)
    B, H, Tq, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H, Tq), dtype=torch.float32, device=q.device)
    if k_sink is not None:
        _need(k_sink, "k_sink", dims=4)
        _need(v_sink, "v_sink", dims=4)
        check("swa_attn_chunk_ring_sink",
              lib().swa_attn_chunk_ring_sink(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring),
                                             _ptr(v_ring), _ptr(k_sink), _ptr(v_sink),
                                             k_sink.shape[2], _ptr(q_start), _ptr(out), _ptr(lse),
                                             B, H, Hkv, Tq, d, W, scale, 1 if update_ring else 0,
                                             _stream(q.device)))
    else:
        check("swa_attn_chunk_ring",
              lib().swa_attn_chunk_ring(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring),
                                        _ptr(v_ring), _ptr(q_start), _ptr(out), _ptr(lse), B, H,
                                        Hkv, Tq, d, W, scale, 1 if update_ring else 0,
                                        _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_attn_chunk_ring_ragged(q, k_new, v_new, k_ring, v_ring, q_start, chunk_len,
                               scale: float | None = None, update_ring: bool = False, out=None,
                               lse=None, return_lse: bool = False):
    """swa_attn_chunk_ring with chunk_len [B] valid rows per sequence (the rest is padding).

    Output rows at or beyond chunk_len[b] are left as they were in `out` (zeros when `out` is
    allocated here), likewise their lse entries.
    """
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_ring, "k_ring"),
                 (v_ring, "v_ring")):
        _need(t, n, dims=4)
    _need(q_start, "q_start", torch.int64, 1)
    _need(chunk_len, "chunk_len", torch.int64, 1)
    B, H, Tq, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.zeros_like(q)
    if return_lse and lse is None:
        lse = torch.zeros((B, H, Tq), dtype=torch.float32, device=q.device)
    check("swa_attn_chunk_ring_ragged",
          lib().swa_attn_chunk_ring_ragged(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring),
                                           _ptr(v_ring), _ptr(q_start), _ptr(chunk_len),
                                           _ptr(out), _ptr(lse), B, H, Hkv, Tq, d, W, scale,
                                           1 if update_ring else 0, _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_chunk_split_workspace_bytes(B: int, H: int, Hkv: int, Tq: int, d: int, W: int) -> int:
    return int(lib().swa_chunk_split_workspace_bytes(B, H, Hkv, Tq, d, W))


def swa_attn_chunk_ring_split(q, k_new, v_new, k_ring, v_ring, q_start, scale: float | None = None,
                              chunk_len=None, k_sink=None, v_sink=None, update_ring: bool = False,
                              out=None, lse=None, return_lse: bool = False, workspace=None):
    """Chunked prefill on a ring cache with a workspace that balances the work.

    The same results as swa_attn_chunk_ring / _ragged (chunk_len [B]) / _sink
    (k_sink, v_sink [B,Hkv,S,d]), within rounding: the last round of units is
    split across the SMs by key range and merged.  Rows past chunk_len[b] keep
    what `out` held (zeros when allocated here).
    """
    for t, n in ((q, "q"), (k_new, "k_new"), (v_new, "v_new"), (k_ring, "k_ring"),
                 (v_ring, "v_ring")):
        _need(t, n, dims=4)
    _need(q_start, "q_start", torch.int64, 1)
    if chunk_len is not None:
        _need(chunk_len, "chunk_len", torch.int64, 1)
    n_sink = 0
    if k_sink is not None:
        _need(k_sink, "k_sink", dims=4)
        _need(v_sink, "v_sink", dims=4)
        n_sink = k_sink.shape[2]
    B, H, Tq, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.zeros_like(q)
    if return_lse and lse is None:
        lse = torch.zeros((B, H, Tq), dtype=torch.float32, device=q.device)
    need = swa_chunk_split_workspace_bytes(B, H, Hkv, Tq, d, W)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check("swa_attn_chunk_ring_split",
          lib().swa_attn_chunk_ring_split(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ring),
                                          _ptr(v_ring), _ptr(k_sink), _ptr(v_sink), n_sink,
                                          _ptr(q_start), _ptr(chunk_len), _ptr(out), _ptr(lse), B,
                                          H, Hkv, Tq, d, W, scale, 1 if update_ring else 0,
                                          _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_ring_write(k_new, v_new, k_ring, v_ring, q_start):
    """Write the chunk rows among the last W positions into slot position mod W (in place)."""
    for t, n in ((k_new, "k_new"), (v_new, "v_new"), (k_ring, "k_ring"), (v_ring, "v_ring")):
        _need(t, n, dims=4)
    _need(q_start, "q_start", torch.int64, 1)
    B, Hkv, T, d = k_new.shape
    W = k_ring.shape[2]
    check("swa_ring_write", lib().swa_ring_write(_ptr(k_new), _ptr(v_new), _ptr(k_ring),
                                                 _ptr(v_ring), _ptr(q_start), B, Hkv, T, d, W,
                                                 _stream(k_new.device)))


def swa_decode_workspace_bytes(B: int, H: int, Hkv: int, d: int, W: int) -> int:
    return int(lib().swa_decode_workspace_bytes(B, H, Hkv, d, W))


def swa_attn_decode_ring(q, k_ring, v_ring, pos, scale: float | None = None, workspace=None,
                         out=None, lse=None, return_lse: bool = False, k_sink=None,
                         v_sink=None):
    """Decode: q [B,H,d] at positions pos [B] over ring caches [B,Hkv,W,d] -> out [B,H,d].

    With k_sink / v_sink [B,Hkv,S,d] (positions 0..S-1) the sinks before the window are
    attended too (swa_attn_decode_ring_sink).
    """
    _need(q, "q", dims=3)
    _need(k_ring, "k_ring", dims=4)
    _need(v_ring, "v_ring", dims=4)
    _need(pos, "pos", torch.int64, 1)
    B, H, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = swa_decode_workspace_bytes(B, H, Hkv, d, W)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    if k_sink is not None:
        _need(k_sink, "k_sink", dims=4)
        _need(v_sink, "v_sink", dims=4)
        check("swa_attn_decode_ring_sink",
              lib().swa_attn_decode_ring_sink(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(k_sink),
                                              _ptr(v_sink), k_sink.shape[2], _ptr(pos), _ptr(out),
                                              _ptr(lse), B, H, Hkv, d, W, scale, _ptr(workspace),
                                              ws_bytes, _stream(q.device)))
    else:
        check("swa_attn_decode_ring",
              lib().swa_attn_decode_ring(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(pos),
                                         _ptr(out), _ptr(lse), B, H, Hkv, d, W, scale,
                                         _ptr(workspace), ws_bytes, _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_attn_decode_ring_static(q, k_ring, v_ring, pos, scale: float | None = None, out=None,
                                lse=None, return_lse: bool = False):
    """Decode like swa_attn_decode_ring, for callers that cannot provide device scratch.

    The library keeps the split partials in its own fixed 16 MiB device array,
    so nothing is allocated for scratch; larger requests raise SwaError
    (SWA_ERR_WORKSPACE).
    Calls on one device share that array: do not let two of them overlap on
    the GPU (keep them on one stream or order them with events).  The first
    call on a device resolves the array's address; make it before any stream
    capture.
    """
    _need(q, "q", dims=3)
    _need(k_ring, "k_ring", dims=4)
    _need(v_ring, "v_ring", dims=4)
    _need(pos, "pos", torch.int64, 1)
    B, H, d = q.shape
    Hkv, W = k_ring.shape[1], k_ring.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if return_lse and lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    check("swa_attn_decode_ring_static",
          lib().swa_attn_decode_ring_static(_ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(pos),
                                            _ptr(out), _ptr(lse), B, H, Hkv, d, W, scale,
                                            _stream(q.device)))
    return (out, lse) if return_lse else out


def swa_ring_slot_positions(n_written, W: int, out=None):
    """int64 [B, W]: the logical position each ring slot holds after n_written[b] writes (-1 empty)."""
    _need(n_written, "n_written", torch.int64, 1)
    B = n_written.numel()
    if out is None:
        out = torch.empty((B, W), dtype=torch.int64, device=n_written.device)
    check("swa_ring_slot_positions", lib().swa_ring_slot_positions(
        B, _ptr(n_written), W, _ptr(out), _stream(n_written.device)))
    return out


def swa_selftest_wait(limit_ns: int, arrive: bool = False, device=None):
    """Run the library's bounded device wait in a one-CTA kernel of its own.

    arrive=False: nobody arrives on the barrier, so the wait gives up after
    limit_ns and swa_get_device_status() then reports SWA_ERR_TIMEOUT (5).
    Returns int32 [5] on the device: lanes of warps 0..3 whose wait succeeded,
    then the elapsed microseconds.
    """
    device = torch.device("cuda") if device is None else torch.device(device)
    res = torch.zeros(5, dtype=torch.int32, device=device)
    check("swa_selftest_wait", lib().swa_selftest_wait(int(limit_ns), 1 if arrive else 0,
                                                       _ptr(res), _stream(device)))
    return res


def swa_get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word as a status code."""
    s = _stream() if stream is None else stream
    return int(lib().swa_get_device_status(s))


def swa_attn_fwd_seq_parallel(q, k, v, W: int, scale: float | None = None, out=None,
                              return_lse: bool = False, group=None, ring_k=None, ring_v=None):
    """Prefill of a sequence split along its length across ranks (see ``seq_parallel``)."""
    from .seq_parallel import swa_attn_fwd_seq_parallel as run

    return run(q, k, v, W, scale=scale, out=out, return_lse=return_lse, group=group,
               ring_k=ring_k, ring_v=ring_v)
