"""swa_attn_varlen (packed sequences, per-sequence windows) and sinks vs the oracle.

Outputs are compared with assert_close_bf16out: the 1e-2 max-abs bar plus the
bf16 rounding of each output value (these cases include rows with only two or
three visible keys, whose outputs reach |o| ~ 2.5).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from tests._util import assert_close_bf16out, assert_close_by_keys, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _packed(seed, lens, H, Hkv, d, extra=0):
    """Token-major inputs for the given lengths, plus `extra` tokens after the last sequence."""
    total = sum(lens) + extra
    q = si.normal_bf16(seed, si.STREAM["q"], (total, H, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (total, Hkv, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (total, Hkv, d))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    return q, k, v, cu


def _run(swa, q, k, v, cu, W, scale, n_sink, fill=5.0):
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    out = torch.full_like(tq, fill)
    lse = torch.full((q.shape[1], q.shape[0]), fill, dtype=torch.float32, device="cuda")
    max_len = int(np.max(np.diff(cu))) if len(cu) > 1 else 1
    swa.swa_attn_varlen(tq, tk, tv, tcu, max(max_len, 1), W, scale, n_sink=n_sink, out=out,
                        lse=lse, return_lse=True)
    assert swa.swa_get_device_status() == 0
    return to_f64(out), to_f64(lse)


@pytest.mark.parametrize("lens,H,Hkv,d,W,S", [
    ([300, 1, 129, 0, 517], 8, 2, 128, 256, 0),    # head pairs; empty and one-token sequences
    ([300, 1, 129, 0, 517], 8, 2, 128, 256, 4),    # the same with four sinks
    ([1000, 64, 255], 6, 2, 64, 100, 0),           # odd group: query-tile pairs
    ([1000, 64, 255], 6, 2, 64, 100, 3),
    ([128, 128, 128], 4, 4, 128, 64, 128),         # a full sink tile
    ([700], 4, 1, 128, 1000, 0),                   # window wider than the sequence
    ([333, 90], 2, 1, 128, 1, 2),                  # W = 1 with sinks
])
def test_varlen_full_tensor(swa, lens, H, Hkv, d, W, S):
    seed = 500 + sum(lens) + W + S
    q, k, v, cu = _packed(seed, lens, H, Hkv, d, extra=37)
    scale = 1.0 / math.sqrt(d)
    got, got_lse = _run(swa, q, k, v, cu, W, scale, S)
    n = int(cu[-1])
    ref, ref_lse = oracle.swa_varlen(q[:n], k[:n], v[:n], cu, W, scale, n_sink=S, with_lse=True)
    assert_close_bf16out(got[:n], ref, what=f"varlen lens={lens} W={W} S={S}")
    assert np.max(np.abs(got_lse[:, :n] - ref_lse.T)) < 1e-3
    # tokens after the last sequence are outside every sequence: untouched
    assert np.all(got[n:] == 5.0) and np.all(got_lse[:, n:] == 5.0)


def test_varlen_long_mixed_lengths(swa):
    """Lengths across many tiles with a ragged tail; sampled rows at every boundary."""
    lens = [4096 + 37, 2000, 129, 5000]
    H, Hkv, d, W, S = 8, 2, 128, 1024, 4
    q, k, v, cu = _packed(41, lens, H, Hkv, d)
    got, _ = _run(swa, q, k, v, cu, W, 1.0 / math.sqrt(d), S)
    rng = np.random.default_rng(3)
    toks = set(rng.integers(0, int(cu[-1]), 300).tolist())
    for a, b in zip(cu[:-1], cu[1:]):
        toks |= {int(a), int(a) + 1, int(b) - 1, int(a) + 127, int(a) + 128, int(a) + W,
                 int(a) + W + 1}
    toks = sorted(t for t in toks if 0 <= t < int(cu[-1]))
    rows = np.array([(t, h) for t in toks for h in (0, 3, 7)], dtype=np.int64)
    ref = oracle.swa_varlen(q, k, v, cu, W, 1.0 / math.sqrt(d), n_sink=S, rows=rows)
    assert_close_bf16out(got[rows[:, 0], rows[:, 1]], ref, what="varlen long")


def test_varlen_equal_lengths_match_batched_layout(swa):
    """B sequences of N tokens: the packed result is the [B,H,N,d] one, bit for bit."""
    B, H, Hkv, N, d, W = 3, 8, 2, 640, 128, 256
    q = si.normal_bf16(9, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(9, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(9, si.STREAM["v"], (B, Hkv, N, d))
    for S in (0, 4):
        ref = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, n_sink=S)
        tm = lambda x: torch.from_numpy(x).view(torch.bfloat16).permute(0, 2, 1, 3).reshape(
            B * N, x.shape[1], d).contiguous().cuda()
        cu = torch.arange(0, (B + 1) * N, N, dtype=torch.int64, device="cuda")
        got = swa.swa_attn_varlen(tm(q), tm(k), tm(v), cu, N, W, n_sink=S)
        assert swa.swa_get_device_status() == 0
        assert torch.equal(got.view(B, N, H, d).permute(0, 2, 1, 3), ref)


def test_varlen_bad_offsets_set_device_status(swa):
    """A decreasing cu_seqlens entry is reported on the device; the rest still runs."""
    q, k, v, cu = _packed(5, [200, 100], 4, 2, 64)
    bad = np.array([0, 200, 150], dtype=np.int64)
    tcu = torch.tensor(bad, device="cuda")
    out = torch.zeros_like(to_dev(q))
    swa.swa_attn_varlen(to_dev(q), to_dev(k), to_dev(v), tcu, 200, 64, out=out)
    assert swa.swa_get_device_status() == 6
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_varlen(q[:200], k[:200], v[:200], [0, 200], 64, 0.125)
    assert_close_bf16out(to_f64(out)[:200], ref, what="valid sequence next to a bad one")


@pytest.mark.parametrize("B,H,Hkv,N,d,W,S", [
    (2, 8, 2, 700, 128, 128, 4),    # sink tile ahead of the window
    (1, 4, 4, 300, 128, 200, 4),    # window reaches tile 0 for the later query tiles
    (2, 6, 2, 513, 64, 64, 1),      # query-tile pairs, one sink
    (2, 3, 1, 513, 64, 64, 1),      # G = 3 with H odd, one sink
    (1, 2, 2, 3000, 128, 1500, 4),  # query-tile pairs, a window of twelve key tiles
    (1, 8, 2, 256, 128, 1000, 4),   # window covers everything: sinks change nothing
])
def test_fwd_sink_full_tensor(swa, B, H, Hkv, N, d, W, S):
    seed = 700 + N + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, N, d))
    scale = 1.0 / math.sqrt(d)
    out, lse = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, scale, n_sink=S,
                                return_lse=True)
    assert swa.swa_get_device_status() == 0
    got, got_lse = to_f64(out), to_f64(lse)
    for b in range(B):
        tm = lambda x: np.ascontiguousarray(x[b].transpose(1, 0, 2))
        ref, ref_lse = oracle.swa_varlen(tm(q), tm(k), tm(v), [0, N], W, scale, n_sink=S,
                                         with_lse=True)
        assert_close_bf16out(got[b].transpose(1, 0, 2), ref, what=f"sinks b={b}")
        assert np.max(np.abs(got_lse[b].T - ref_lse)) < 1e-3


def test_varlen_workload_sampled_rows(swa):
    """The benchmarked packed batch (16 sequences of 256..16384 tokens), sampled rows."""
    from swa_inputs.workloads import WORKLOADS, varlen_inputs

    w = WORKLOADS["varlen_prefill"]
    q, k, v, cu = varlen_inputs(w)
    got, _ = _run(swa, q, k, v, cu, w.W, w.scale, w.n_sink)
    rng = np.random.default_rng(8)
    toks = set(rng.integers(0, int(cu[-1]), 200).tolist())
    for a, b in zip(cu[:-1], cu[1:]):
        toks |= {int(a), int(a) + 127, int(a) + 128, int(a) + w.W, int(b) - 1}
    toks = sorted(t for t in toks if 0 <= t < int(cu[-1]))
    rows = np.array([(t, int(rng.integers(w.H))) for t in toks], dtype=np.int64)
    ref = oracle.swa_varlen(q, k, v, cu, w.W, w.scale, n_sink=w.n_sink, rows=rows)
    assert_close_bf16out(got[rows[:, 0], rows[:, 1]], ref, what="varlen workload")


def test_varlen_workload_whole_sequences_every_element(swa):
    """The benchmarked packed batch: every output element (all heads) and the LSE of
    each sequence of at most 4096 tokens and of the longest one, in the call that
    packs all sixteen."""
    from swa_inputs.workloads import WORKLOADS, varlen_inputs

    w = WORKLOADS["varlen_prefill"]
    q, k, v, cu = varlen_inputs(w)
    got, got_lse = _run(swa, q, k, v, cu, w.W, w.scale, w.n_sink)
    lens = np.diff(cu)
    short = [s for s in range(len(lens)) if lens[s] <= 4096]
    assert short
    for s in short + [int(np.argmax(lens))]:
        a, e = int(cu[s]), int(cu[s + 1])
        ref, ref_lse = oracle.swa_varlen(q[a:e], k[a:e], v[a:e], [0, e - a], w.W, w.scale,
                                         n_sink=w.n_sink, with_lse=True)
        keys = np.minimum(np.arange(e - a) + 1, w.W)[:, None]
        assert_close_by_keys(got[a:e], ref, keys, what=f"varlen workload seq {s} ({e - a} tokens)")
        assert np.max(np.abs(got_lse[:, a:e] - ref_lse.T)) < 1e-3  # kernel LSE is [H, total]


def test_sink_prefill_workload_sampled_rows(swa):
    """The benchmarked Mistral-shaped prefill with 4 sinks, sampled rows (tile edges included)."""
    from swa_inputs.workloads import WORKLOADS, prefill_inputs

    w = WORKLOADS["mistral_prefill_sink"]
    q, k, v = prefill_inputs(w)
    out = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), w.W, w.scale, n_sink=w.n_sink)
    assert swa.swa_get_device_status() == 0
    got = to_f64(out)
    tm = lambda x: np.ascontiguousarray(x[0].transpose(1, 0, 2))
    rng = np.random.default_rng(9)
    toks = sorted(set(rng.integers(0, w.N, 200).tolist()) |
                  {0, 1, 127, 128, w.W - 1, w.W, w.W + 1, w.W + 3, w.W + 4, w.N - 1})
    rows = np.array([(t, int(rng.integers(w.H))) for t in toks], dtype=np.int64)
    ref = oracle.swa_varlen(tm(q), tm(k), tm(v), [0, w.N], w.W, w.scale, n_sink=w.n_sink,
                            rows=rows)
    assert_close_bf16out(got[0, rows[:, 1], rows[:, 0]], ref, what="sink prefill workload")
