"""Sequence-parallel prefill: every rank holds a contiguous slice of the sequence.

A query at position i reads keys i - W + 1 .. i, so the rank holding rows
[start, start + n) needs, besides its own keys, only the W - 1 key/value rows
before ``start`` (fewer near the sequence start).  Those rows (the halo) come
from the ranks holding them, in one round of point-to-point sends; no other
data crosses ranks and there is no reduction.  The halo is written into a
W-slot ring cache (slot = position mod W) by ``swa_ring_write``, and the
shard is then exactly a chunked prefill at ``q_start = start``
(``swa_attn_chunk_ring``): the ring supplies the positions before the shard,
the shard's own K/V the rest.  All attention arithmetic runs in the CUDA
kernels; this module only moves rows between ranks and lays them out.

Sources: the window rule of the M003 note "weight sparsity vs attention
sparsity", section 03, and Chapter 10 "local and sparse attention: SWA and
DSA", section 10.1 (a query sees itself and the W - 1 positions before it);
Chapter 10 section 10.2 (a chunk of queries needs keys from before the chunk,
held in the rolling cache of the "Dense attention vs sparse SWA" blog,
section 3.2).
"""

from __future__ import annotations

import math
from typing import Sequence

import torch
import torch.distributed as dist


def shard_starts(lengths: Sequence[int]) -> list[int]:
    """First sequence position of each rank's shard (shards in rank order)."""
    starts, s = [], 0
    for n in lengths:
        if n < 0:
            raise ValueError("shard lengths must be >= 0")
        starts.append(s)
        s += int(n)
    return starts


def halo_plan(lengths: Sequence[int], W: int) -> list[tuple[int, int, int, int]]:
    """Rows each rank sends for the others' halos, as (src, dst, lo, hi).

    Rank ``dst`` (first position ``start``) needs positions
    ``max(0, start - W + 1) .. start - 1``; rank ``src`` sends its local rows
    ``lo .. hi - 1`` of them.  Entries are ordered by ``dst``, then by
    ascending position, so concatenating what ``dst`` receives in plan order
    gives its halo in position order.
    """
    if W < 1:
        raise ValueError("W must be >= 1")
    starts = shard_starts(lengths)
    plan = []
    for dst, start in enumerate(starts):
        need_lo, need_hi = max(0, start - (W - 1)), start
        for src in range(dst):
            lo = max(need_lo, starts[src])
            hi = min(need_hi, starts[src] + int(lengths[src]))
            if lo < hi:
                plan.append((src, dst, lo - starts[src], hi - starts[src]))
    return plan


def exchange_halo(k: torch.Tensor, v: torch.Tensor, W: int, group=None):
    """Gather this rank's halo: the K/V rows of the W - 1 positions before its shard.

    k, v: this rank's shard ``[B, Hkv, n, d]`` (shards in rank order along the
    sequence; n may differ between ranks).  Returns ``(start, halo_k, halo_v)``
    with halo rows ``[B, Hkv, h, d]`` for positions ``start - h .. start - 1``,
    h = min(W - 1, start).  One all-gather of the shard lengths, then one
    batch of sends and receives.  Works on any backend whose point-to-point
    ops accept the tensors' device (NCCL for CUDA tensors, gloo for CPU);
    with NCCL, set each rank's current CUDA device before the first call.
    Every rank of the group must call it with the same W.
    """
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    B, Hkv, n, d = k.shape
    if v.shape != k.shape:
        raise ValueError("k and v must have the same shape")
    mine = torch.tensor([n], dtype=torch.int64, device=k.device)
    every = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(every, mine, group=group)
    lengths = [int(t.item()) for t in every]
    start = shard_starts(lengths)[rank]
    plan = halo_plan(lengths, W)

    def peer(r):
        return r if group is None else dist.get_global_rank(group, r)

    ops, pieces = [], []
    for src, dst, lo, hi in plan:
        if src == rank:
            for t in (k, v):
                ops.append(dist.P2POp(dist.isend, t[:, :, lo:hi].contiguous(), peer(dst),
                                      group))
        elif dst == rank:
            pk = torch.empty((B, Hkv, hi - lo, d), dtype=k.dtype, device=k.device)
            pv = torch.empty_like(pk)
            ops.append(dist.P2POp(dist.irecv, pk, peer(src), group))
            ops.append(dist.P2POp(dist.irecv, pv, peer(src), group))
            pieces.append((pk, pv))
    if ops:
        for work in dist.batch_isend_irecv(ops):
            work.wait()
    if pieces:
        halo_k = torch.cat([p[0] for p in pieces], dim=2)
        halo_v = torch.cat([p[1] for p in pieces], dim=2)
    else:
        halo_k = k.new_empty((B, Hkv, 0, d))
        halo_v = v.new_empty((B, Hkv, 0, d))
    if halo_k.shape[2] != min(W - 1, start):
        raise RuntimeError("halo rows do not cover the window before this shard")
    return start, halo_k, halo_v


def shard_attention(q, k, v, halo_k, halo_v, start: int, W: int,
                    scale: float | None = None, out=None, return_lse: bool = False,
                    ring_k=None, ring_v=None):
    """Attention of one shard given its halo (no communication).

    q ``[B, H, n, d]`` at positions ``start .. start + n - 1``; k, v the
    shard's own rows; halo_k, halo_v ``[B, Hkv, h, d]`` the positions
    ``start - h .. start - 1`` with h = min(W - 1, start).  Optional ring
    buffers ``[B, Hkv, W, d]`` are overwritten (zeroed, then the halo
    written); by default they are allocated.  Returns what
    ``swa_attn_chunk_ring`` returns: rows identical in meaning to rows
    ``start ..`` of a prefill over the whole sequence.
    """
    from . import swa_attn_chunk_ring, swa_ring_write

    B, Hkv, n, d = k.shape
    h = halo_k.shape[2]
    if h != min(W - 1, start):
        raise ValueError(f"halo has {h} rows, the window needs {min(W - 1, start)}")
    if n == 0:  # an empty shard has no rows to compute
        o = torch.empty_like(q) if out is None else out
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        return (o, lse) if return_lse else o
    if ring_k is None:
        ring_k = torch.zeros((B, Hkv, W, d), dtype=k.dtype, device=k.device)
        ring_v = torch.zeros_like(ring_k)
    else:
        # slots the halo does not fill hold positions no query of the shard can
        # see; they still enter the tile MMAs, so they must be finite
        ring_k.zero_()
        ring_v.zero_()
    if h:
        first = torch.full((B,), start - h, dtype=torch.int64, device=k.device)
        swa_ring_write(halo_k.contiguous(), halo_v.contiguous(), ring_k, ring_v, first)
    q_start = torch.full((B,), start, dtype=torch.int64, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    return swa_attn_chunk_ring(q, k, v, ring_k, ring_v, q_start, scale=scale, out=out,
                               return_lse=return_lse)


def swa_attn_fwd_seq_parallel(q, k, v, W: int, scale: float | None = None, out=None,
                              return_lse: bool = False, group=None, ring_k=None,
                              ring_v=None):
    """Prefill of a sequence split along its length across the ranks of ``group``.

    Rank r holds q ``[B, H, n_r, d]`` and k, v ``[B, Hkv, n_r, d]`` for
    positions ``sum(n_0 .. n_{r-1}) ..``; the output rows are those of
    ``swa_attn_fwd`` over the whole sequence.  Every rank must call it (the
    halo exchange is collective).
    """
    start, halo_k, halo_v = exchange_halo(k, v, W, group)
    return shard_attention(q, k, v, halo_k, halo_v, start, W, scale=scale, out=out,
                           return_lse=return_lse, ring_k=ring_k, ring_v=ring_v)
