"""swa_attn_fwd (tile-skipping prefill) against the fp64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from swa_inputs.workloads import WORKLOADS, prefill_inputs
from tests._util import assert_close, sample_rows, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _inputs(seed, B, H, Hkv, N, d):
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, N, d))
    return q, k, v


def _run(swa, q, k, v, W, scale, lse=False):
    r = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, scale, return_lse=lse)
    assert swa.swa_get_device_status() == 0
    return r


def test_tiny_workload_full_tensor(swa):
    w = WORKLOADS["tiny"]
    q, k, v = prefill_inputs(w)
    out, lse = _run(swa, q, k, v, w.W, w.scale, lse=True)
    ref, ref_lse = oracle.swa_forward(q, k, v, w.W, w.scale, with_lse=True)
    assert_close(to_f64(out), ref, what="tiny")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3


@pytest.mark.parametrize("B,H,Hkv,N,d,W", [
    (1, 2, 2, 128, 128, 128),   # one tile, full causal
    (1, 2, 1, 256, 128, 100),   # GQA, window inside tiles
    (2, 4, 2, 200, 128, 64),    # ragged tail
    (1, 4, 4, 129, 64, 1),      # W = 1
    (1, 2, 2, 1, 128, 5),       # single row
    (1, 8, 2, 640, 128, 128),   # window == tile
    (1, 8, 2, 640, 128, 129),
    (1, 8, 2, 640, 128, 127),
    (1, 2, 2, 300, 64, 10000),  # W >> N: full causal
    (1, 4, 1, 1000, 128, 333),
])
def test_small_shapes_full_tensor(swa, B, H, Hkv, N, d, W):
    q, k, v = _inputs(100 + N + W, B, H, Hkv, N, d)
    scale = 1.0 / math.sqrt(d)
    out = _run(swa, q, k, v, W, scale)
    ref = oracle.swa_forward(q, k, v, W, scale)
    assert_close(to_f64(out), ref, what=f"B{B} H{H}/{Hkv} N{N} d{d} W{W}")


@pytest.mark.parametrize("B,H,Hkv,N,d,W", [
    (1, 6, 2, 700, 128, 200),    # G = 3
    (2, 2, 2, 1000, 128, 1024),  # eight-tile window
    (1, 2, 2, 1000, 128, 1025),  # one more key
    (1, 3, 3, 500, 64, 300),     # H odd
    (1, 6, 6, 333, 64, 77),      # d = 64, ragged tail
    (3, 4, 4, 130, 128, 129),    # two query tiles, the second of two rows
])
def test_query_tile_pairs_for_odd_groups(swa, B, H, Hkv, N, d, W):
    """With G = H / Hkv odd a unit is query tiles 2p and 2p + 1 of one head
    (the key stream is the union of both windows); against the oracle, with
    the log-sum-exp."""
    q, k, v = _inputs(300 + N + W, B, H, Hkv, N, d)
    scale = 1.0 / math.sqrt(d)
    out, lse = _run(swa, q, k, v, W, scale, lse=True)
    ref, ref_lse = oracle.swa_forward(q, k, v, W, scale, with_lse=True)
    assert_close(to_f64(out), ref, what=f"B{B} H{H}/{Hkv} N{N} d{d} W{W}")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3


def test_worked_example_zero_scores(swa):
    """M003 note section 05: zero scores, V = 1..8 -> 7 (W = 3) and 4.5 (full)."""
    N, d = 8, 64
    q = np.zeros((1, 1, N, d), dtype=np.uint16)  # bf16 zero
    k = si.normal_bf16(1, 2, (1, 1, N, d))
    vals = np.zeros((1, 1, N, d), dtype=np.float32)
    vals[0, 0, :, 0] = np.arange(1, 9)
    v = si.f32_to_bf16_bits(vals)
    out3 = to_f64(_run(swa, q, k, v, 3, 0.125))
    outf = to_f64(_run(swa, q, k, v, 8, 0.125))
    assert abs(out3[0, 0, 7, 0] - 7.0) < 1e-6
    assert abs(outf[0, 0, 7, 0] - 4.5) < 1e-6


@pytest.mark.parametrize("name", ["mistral_prefill", "narrow_window"])
def test_workload_sampled_rows(swa, name):
    w = WORKLOADS[name]
    q, k, v = prefill_inputs(w)
    out = _run(swa, q, k, v, w.W, w.scale)
    # the first and last row of every query tile, and the rows around the window
    # edge (W - 2 .. W) and the last row, each at a random (b, h); sample_rows
    # keeps every listed row
    edges = []
    for t in range(0, w.N, 128):
        edges += [t, t + 127]
    edges += [w.W - 2, w.W - 1, w.W, w.N - 1]
    rows = sample_rows(w.B, w.H, w.N, 384, seed=7, extra=edges)
    listed = set(int(i) for i in rows[:, 2])
    assert all(i in listed for i in edges)
    ref = oracle.swa_forward(q, k, v, w.W, w.scale, rows=rows)
    got = to_f64(out)[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_close(got, ref, what=name)
    # relative RMS error: outputs here are ~0.02 in size, so also bound the error
    # relative to them (bf16 rounding of the output alone is ~2^-9 relative)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-2


@pytest.mark.parametrize("W,needle", [(64, 100), (64, 127), (64, 128), (512, 511), (512, 512),
                                      (512, 1000), (4096, 4095), (4096, 4096), (4096, 1)])
def test_needle_window_boundary(swa, W, needle):
    """One key dominates every score it enters; a query sees it iff the needle
    position lies in [i - W + 1, i], so an off-by-one window changes O(1) values."""
    N, d = max(2 * W + 256, 1024), 128
    u = np.zeros(d, dtype=np.float32)
    u[:8] = 1.0
    qf = np.tile(u, (1, 1, N, 1))
    kf = si.bf16_bits_to_f32(si.normal_bf16(5, 2, (1, 1, N, d))) * 0.1
    kf[0, 0, needle] = 8.0 * u / np.linalg.norm(u) * math.sqrt(d)
    vf = si.bf16_bits_to_f32(si.normal_bf16(5, 3, (1, 1, N, d)))
    q, k, v = (si.f32_to_bf16_bits(x.astype(np.float32)) for x in (qf, kf, vf))
    scale = 1.0 / math.sqrt(d)
    out = to_f64(_run(swa, q, k, v, W, scale))[0, 0]
    ref = oracle.swa_forward(q, k, v, W, scale)[0, 0]
    assert_close(out, ref, what="needle")
    vneedle = si.bf16_bits_to_f32(v)[0, 0, needle].astype(np.float64)
    for i in [needle - 1, needle, needle + W - 1, needle + W]:
        if 0 <= i < N:
            sees = needle <= i <= needle + W - 1
            close = np.max(np.abs(out[i] - vneedle)) < 0.05
            assert close == sees, f"query {i}: sees needle {sees}, output matches {close}"


def test_chunk_of_rows_matches_causal_prefix(swa):
    """Future values do not change past outputs (Chapter 10 section 10.5)."""
    B, H, Hkv, N, d, W = 1, 4, 2, 512, 128, 100
    q, k, v = _inputs(42, B, H, Hkv, N, d)
    a = _run(swa, q, k, v, W, 0.1)
    v2 = v.copy()
    v2[:, :, 300:] = si.normal_bf16(43, 3, v2[:, :, 300:].shape)
    b = _run(swa, q, k, v2, W, 0.1)
    assert torch.equal(a[:, :, :300], b[:, :, :300])
