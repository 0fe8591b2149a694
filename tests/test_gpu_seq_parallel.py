"""Sequence-parallel prefill on one GPU: every shard of a sequence in turn.

The ranks are emulated one after the other in this process: shard r's halo is
assembled from the other shards' rows exactly as the exchange plan sends them
(the exchange itself is tested on gloo ranks on the CPU), then
``shard_attention`` writes it into a ring with ``swa_ring_write`` and runs
``swa_attn_chunk_ring``.  Every shard's output must match the oracle's
prefill over the whole sequence (same rows), and the prefill kernel over the
whole sequence within the same tolerance.  Ring buffers are reused across
shards, so stale slots from the previous shard must not leak.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from sliding_window_sparse_b200.seq_parallel import halo_plan, shard_attention, shard_starts
from tests._util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


@pytest.mark.parametrize("B,H,Hkv,d,W,lengths", [
    (1, 8, 2, 128, 300, [137, 400, 63, 0, 400]),   # one halo spans two shards; empty shard
    (2, 4, 4, 64, 128, [256, 256, 256]),           # aligned shards, shards longer than W
    (1, 4, 1, 128, 1000, [300, 300, 300]),         # window longer than every shard
])
def test_shards_match_whole_sequence(swa, B, H, Hkv, d, W, lengths):
    n = sum(lengths)
    seed = 500 + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, n, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, n, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, n, d))
    scale = 1.0 / math.sqrt(d)
    ref = oracle.swa_forward(q, k, v, W, scale).reshape(B, H, n, d)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    whole = to_f64(swa.swa_attn_fwd(tq, tk, tv, W, scale))
    starts = shard_starts(lengths)
    plan = halo_plan(lengths, W)
    ring_k = torch.full((B, Hkv, W, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    ring_v = torch.full_like(ring_k, float("nan"))
    for r, (s0, ln) in enumerate(zip(starts, lengths)):
        parts = [(src, lo, hi) for src, dst, lo, hi in plan if dst == r]
        hk = torch.cat([tk[:, :, starts[s] + lo:starts[s] + hi] for s, lo, hi in parts], 2) \
            if parts else tk[:, :, :0]
        hv = torch.cat([tv[:, :, starts[s] + lo:starts[s] + hi] for s, lo, hi in parts], 2) \
            if parts else tv[:, :, :0]
        sl = slice(s0, s0 + ln)
        out = shard_attention(tq[:, :, sl].contiguous(), tk[:, :, sl].contiguous(),
                              tv[:, :, sl].contiguous(), hk, hv, s0, W, scale,
                              ring_k=ring_k, ring_v=ring_v)
        assert swa.swa_get_device_status() == 0
        if ln == 0:
            continue
        got = to_f64(out)
        assert_close(got, ref[:, :, sl], what=f"shard {r}")
        assert_close(got, whole[:, :, sl], what=f"shard {r} vs whole-sequence kernel")
        assert np.linalg.norm(got - ref[:, :, sl]) / np.linalg.norm(ref[:, :, sl]) < 1e-2


def test_shard_rejects_short_halo(swa):
    B, H, Hkv, d, W = 1, 2, 1, 64, 64
    q = torch.zeros((B, H, 16, d), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((B, Hkv, 16, d), dtype=torch.bfloat16, device="cuda")
    halo = torch.zeros((B, Hkv, 10, d), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        shard_attention(q, k, k, halo, halo, 100, W)   # the window needs 63 rows
