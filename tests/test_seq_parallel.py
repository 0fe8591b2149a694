"""Sequence-parallel prefill, host side: the halo plan and its exchange (CPU, gloo).

A rank holding positions [start, start + n) needs the key/value rows of the
W - 1 positions before ``start`` (fewer near the sequence start), and nothing
else from other ranks (window rule: M003 note section 03, Chapter 10 section
10.1).  The plan is checked against a brute-force enumeration of the needed
positions.  The exchange runs on four gloo ranks with uneven shards (one
shorter than W - 1, so one halo spans two ranks, and one empty): each halo
must equal the full sequence's rows bit for bit.  The attention of each
shard, computed here by the oracle's chunked prefill over a ring that holds
the halo, must equal the oracle's prefill over the whole sequence: this pins
how the halo is laid out in the ring (Chapter 10 section 10.2).
"""

import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from sliding_window_sparse_b200.seq_parallel import halo_plan, shard_starts  # noqa: E402

LENGTHS = [37, 5, 0, 26]   # shard 1 is shorter than W - 1; shard 2 is empty
W = 9
B, H, HKV, D = 1, 4, 2, 16


def _brute_needed(lengths, W):
    """For every rank, the (src, position) pairs it must receive, by enumeration."""
    owner = {}
    pos = 0
    for r, n in enumerate(lengths):
        for _ in range(n):
            owner[pos] = r
            pos += 1
    need = []
    start = 0
    for r, n in enumerate(lengths):
        need.append([(owner[p], p) for p in range(start) if start - p <= W - 1])
        start += n
    return need


@pytest.mark.parametrize("lengths,w", [
    ([4, 4, 4], 3), ([2, 2, 2, 2], 6), ([5, 0, 3], 4), ([8, 8], 1), ([3, 7, 1, 9, 2], 5),
    ([100], 50), ([1, 1, 1, 1, 1, 1], 100), (LENGTHS, W),
])
def test_halo_plan_matches_enumeration(lengths, w):
    plan = halo_plan(lengths, w)
    starts = shard_starts(lengths)
    got = [[] for _ in lengths]
    for src, dst, lo, hi in plan:
        assert src < dst and 0 <= lo < hi <= lengths[src]
        got[dst] += [(src, starts[src] + i) for i in range(lo, hi)]
    assert got == _brute_needed(lengths, w)   # same rows, in position order


def test_halo_plan_rejects_bad_window():
    with pytest.raises(ValueError):
        halo_plan([4, 4], 0)
    with pytest.raises(ValueError):
        shard_starts([3, -1])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits_to_torch(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def _torch_to_bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _full_inputs():
    import swa_inputs as si

    n = sum(LENGTHS)
    q = si.normal_bf16(21, si.STREAM["q"], (B, H, n, D))
    k = si.normal_bf16(21, si.STREAM["k"], (B, HKV, n, D))
    v = si.normal_bf16(21, si.STREAM["v"], (B, HKV, n, D))
    return q, k, v


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    from sliding_window_sparse_b200.seq_parallel import exchange_halo

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        q, k, v = _full_inputs()
        s0 = shard_starts(LENGTHS)[rank]
        s1 = s0 + LENGTHS[rank]
        k_loc = _bits_to_torch(k[:, :, s0:s1])
        v_loc = _bits_to_torch(v[:, :, s0:s1])
        start, hk, hv = exchange_halo(k_loc, v_loc, W)
        np.save(os.path.join(out_dir, f"hk{rank}.npy"), _torch_to_bits(hk))
        np.save(os.path.join(out_dir, f"hv{rank}.npy"), _torch_to_bits(hv))
        with open(os.path.join(out_dir, f"start{rank}.txt"), "w") as f:
            f.write(str(start))
    finally:
        dist.destroy_process_group()


def test_gloo_halo_exchange_and_ring_layout(tmp_path):
    import oracle

    world, port = len(LENGTHS), _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    q, k, v = _full_inputs()
    scale = 1.0 / np.sqrt(D)
    full = oracle.swa_forward(q, k, v, W, scale)
    starts = shard_starts(LENGTHS)
    for r in range(world):
        start = int(open(tmp_path / f"start{r}.txt").read())
        assert start == starts[r]
        hk = np.load(tmp_path / f"hk{r}.npy")
        hv = np.load(tmp_path / f"hv{r}.npy")
        h = min(W - 1, start)
        assert hk.shape == (B, HKV, h, D)
        assert np.array_equal(hk, k[:, :, start - h:start])   # bit-exact rows
        assert np.array_equal(hv, v[:, :, start - h:start])
        if LENGTHS[r] == 0:
            continue
        # the shard as a chunked prefill over a ring holding the halo
        ring_k = np.zeros((B, HKV, W, D), dtype=np.uint16)
        ring_v = np.zeros_like(ring_k)
        if h:
            ring_k, ring_v = oracle.ring_update(hk, hv, ring_k, ring_v,
                                                np.full(B, start - h, np.int64), W)
        s1 = start + LENGTHS[r]
        shard = oracle.swa_chunk(q[:, :, start:s1], k[:, :, start:s1], v[:, :, start:s1],
                                 ring_k, ring_v, np.full(B, start, np.int64), W, scale)
        ref = full.reshape(B, H, -1, D)[:, :, start:s1]
        assert np.abs(shard.reshape(ref.shape) - ref).max() <= 1e-12


def _subgroup_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    from sliding_window_sparse_b200.seq_parallel import exchange_halo

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        members = [1, 2, 3]            # global rank 0 takes no part in the exchange
        group = dist.new_group(members)
        if rank in members:
            lengths = [6, 3, 10]       # shard of group rank r = members.index(rank)
            gr = members.index(rank)
            q, k, v = _full_inputs()
            s0 = sum(lengths[:gr])
            k_loc = _bits_to_torch(k[:, :, s0:s0 + lengths[gr]])
            v_loc = _bits_to_torch(v[:, :, s0:s0 + lengths[gr]])
            start, hk, hv = exchange_halo(k_loc, v_loc, W, group=group)
            np.save(os.path.join(out_dir, f"g_hk{gr}.npy"), _torch_to_bits(hk))
            with open(os.path.join(out_dir, f"g_start{gr}.txt"), "w") as f:
                f.write(str(start))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_gloo_halo_exchange_in_a_subgroup(tmp_path):
    """Group ranks are mapped to global ranks for the point-to-point sends."""
    world, port = 4, _free_port()
    mp.spawn(_subgroup_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    _, k, _ = _full_inputs()
    for gr, start in enumerate([0, 6, 9]):
        assert int(open(tmp_path / f"g_start{gr}.txt").read()) == start
        h = min(W - 1, start)
        assert np.array_equal(np.load(tmp_path / f"g_hk{gr}.npy"), k[:, :, start - h:start])
