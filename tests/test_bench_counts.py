"""The work counts behind bench.py's numbers (CPU).

``value`` is useful work over time, so a slip in the counting would inflate
the reported throughput with every kernel still correct.  The counts are
pinned here to the figures the pages fix (21 pairs for N=8, W=3 in the M003
note section 03; the closed form N*W - W*(W-1)/2), to the oracle's
pair enumeration (independent code), and to the workload sizes' own
arithmetic: the Mistral-shaped prefill has 25 167 872 visible pairs per
head, the narrow window 16 646 400 per (batch, head), a 512-row chunk on a
full 4096-slot ring 512 * 4096 per head, and the decode ring holds
2 * 64 * 8 * 4096 * 128 bf16 values of K and V.
"""

import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from swa_inputs.workloads import WORKLOADS, seq_lens  # noqa: E402


def test_worked_example():
    assert bench.sequence_pairs(8, 3) == 21          # M003 note section 03
    assert bench.sequence_pairs(8, 8) == 36          # full causal
    assert bench.sequence_pairs(8, 100) == 36        # W >= N is full causal


@pytest.mark.parametrize("N", [1, 2, 7, 64, 100, 129, 300])
@pytest.mark.parametrize("W", [1, 2, 5, 64, 128, 1000])
@pytest.mark.parametrize("S", [0, 1, 4, 9])
def test_sequence_pairs_matches_enumeration(N, W, S):
    assert bench.sequence_pairs(N, W, S) == oracle.count_pairs_sink(N, W, S)
    if S == 0:
        assert bench.sequence_pairs(N, W) == oracle.count_pairs(N, W)


def test_prefill_counts_at_workload_sizes():
    assert bench.sequence_pairs(512, 64) == 30752
    assert bench.sequence_pairs(8192, 4096) == 25167872 == oracle.count_pairs(8192, 4096)
    assert bench.sequence_pairs(32768, 512) == 16646400
    m = WORKLOADS["mistral_prefill"]
    assert bench.useful_flops(m) == 4 * 128 * 32 * 25167872          # 412.35 GFLOP
    n = WORKLOADS["narrow_window"]
    assert bench.useful_flops(n) == 4 * 128 * 32 * 2 * 16646400      # 545.47 GFLOP
    # the backward counts five products per pair against the forward's two
    assert bench.useful_flops(WORKLOADS["mistral_backward"]) * 2 == bench.useful_flops(m) * 5
    s = WORKLOADS["mistral_prefill_sink"]
    assert bench.useful_flops(s) == 4 * 128 * 32 * oracle.count_pairs_sink(8192, 4096, 4)


def test_chunk_counts():
    c = WORKLOADS["chunk_ring"]
    # q_start = 12288 >= W: every query of the chunk sees a full window
    assert bench.useful_flops(c) == 4 * 128 * 32 * 4 * 512 * 4096    # 137.44 GFLOP
    cs = WORKLOADS["chunk_ring_sink"]
    assert bench.useful_flops(cs) == 4 * 128 * 32 * 4 * 512 * (4096 + 4)
    cr = WORKLOADS["chunk_ring_ragged"]
    lens = [int(x) for x in seq_lens(cr)]
    assert len(lens) == 4 and all(1 <= x <= 512 for x in lens)
    assert bench.useful_flops(cr) == 4 * 128 * 32 * sum(lens) * 4096


def test_chunk_counts_as_rows_of_a_prefill():
    """A chunk's pairs are rows q_start.. of a prefill over q_start + T positions."""
    small = dict(WORKLOADS["chunk_ring"].__dict__)
    for qs, T, W, S in [(0, 37, 16, 0), (5, 20, 16, 2), (40, 9, 16, 3), (100, 64, 32, 0)]:
        small.update(q_start=qs, Tq=T, W=W, n_sink=S, B=1, H=1, d=1, len_hi=0)
        w = type(WORKLOADS["chunk_ring"])(**small)
        want = oracle.count_pairs_sink(qs + T, W, S) - oracle.count_pairs_sink(qs, W, S)
        assert bench.useful_flops(w) == 4 * want


def test_varlen_counts():
    v = WORKLOADS["varlen_prefill"]
    lens = [int(x) for x in seq_lens(v)]
    assert len(lens) == 16 and all(256 <= x <= 16384 for x in lens)
    assert bench.useful_flops(v) == 4 * 128 * 32 * sum(bench.sequence_pairs(n, 4096) for n in lens)
    # the packed backward: five products per visible pair (window and sinks), per sequence
    vb = WORKLOADS["varlen_backward"]
    lens_b = [int(x) for x in seq_lens(vb)]
    assert len(lens_b) == 16 and all(256 <= x <= 16384 for x in lens_b)
    assert bench.useful_flops(vb) == 10 * 128 * 32 * sum(oracle.count_pairs_sink(n, 4096, 4)
                                                         for n in lens_b)


def test_decode_bytes():
    d = WORKLOADS["decode_ring"]
    assert bench.decode_kv_bytes(d) == 1073741824 == 2 * 64 * 8 * 4096 * 128 * 2
    ds = WORKLOADS["decode_ring_sink"]
    pos = bench.decode_positions(ds)
    # sink rows read besides the ring: positions j < 4 before each query's window
    extra = sum(sum(1 for j in range(4) if j < int(p) - 4096 + 1) for p in pos)
    assert bench.decode_kv_bytes(ds) == 2 * 8 * 128 * 2 * (64 * 4096 + extra)
    assert np.all((pos >= 4095) & (pos <= 131071))


def test_algorithmic_bytes():
    m = WORKLOADS["mistral_prefill"]
    q = 32 * 8192 * 128 * 2
    kv = 8 * 8192 * 128 * 2
    assert bench.algorithmic_bytes(m) == 2 * q + 2 * kv == 167772160   # Q + O + K + V
    c = WORKLOADS["chunk_ring"]
    rows = 4 * 512
    assert bench.algorithmic_bytes(c) == 2 * 128 * (2 * 32 * rows + 2 * 8 * (rows + 4 * 4096))
    d = WORKLOADS["decode_ring"]
    assert bench.algorithmic_bytes(d) == 1073741824 + 2 * 128 * 64 * 32 * 2
