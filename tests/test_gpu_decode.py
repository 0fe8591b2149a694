"""swa_attn_decode_ring (split-K decode from a ring cache) against the oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from swa_inputs.workloads import WORKLOADS, decode_inputs
from tests._util import assert_close, assert_close_bf16out, to_dev, to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _run(swa, q, rk, rv, pos, scale, workspace=None):
    out, lse = swa.swa_attn_decode_ring(to_dev(q), to_dev(rk), to_dev(rv),
                                        torch.tensor(pos, dtype=torch.int64, device="cuda"),
                                        scale, workspace=workspace, return_lse=True)
    assert swa.swa_get_device_status() == 0
    return to_f64(out), to_f64(lse)


@pytest.mark.parametrize("B,H,Hkv,d,W,pos", [
    (2, 8, 2, 128, 256, [1000, 255]),           # full windows, G = 4
    (3, 4, 4, 64, 100, [0, 5, 99]),             # partly filled ring, G = 1
    (2, 16, 2, 128, 1000, [5000, 999]),         # G = 8, W not a power of two
    (1, 4, 2, 64, 4096, [70000]),               # G = 2
    (4, 32, 8, 128, 4096, [4095, 4096, 131071, 10]),
])
def test_decode_small_full(swa, B, H, Hkv, d, W, pos):
    seed = 500 + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, d))
    rk = si.normal_bf16(seed, si.STREAM["k_ring"], (B, Hkv, W, d))
    rv = si.normal_bf16(seed, si.STREAM["v_ring"], (B, Hkv, W, d))
    scale = 1.0 / math.sqrt(d)
    out, lse = _run(swa, q, rk, rv, pos, scale)
    ref, ref_lse = oracle.swa_decode(q, rk, rv, pos, W, scale, with_lse=True)
    assert_close(out, ref, what="decode")
    assert np.max(np.abs(lse - ref_lse)) < 1e-3


def test_decode_workload_all_rows(swa):
    w = WORKLOADS["decode_ring"]
    q, rk, rv, pos = decode_inputs(w)
    out, _ = _run(swa, q, rk, rv, list(pos), w.scale)
    ref = oracle.swa_decode(q, rk, rv, pos, w.W, w.scale)
    assert_close(out, ref, what="decode workload")


def test_decode_equals_prefill_last_row(swa):
    """Decode at position p == row p of a prefill over the same keys and values."""
    B, H, Hkv, d, W, N = 2, 8, 2, 128, 300, 777
    q = si.normal_bf16(8, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(8, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(8, si.STREAM["v"], (B, Hkv, N, d))
    full = to_f64(swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, 0.09))
    rk = torch.zeros((B, Hkv, W, d), dtype=torch.bfloat16, device="cuda")
    rv = torch.zeros_like(rk)
    swa.swa_ring_write(to_dev(k), to_dev(v), rk, rv, torch.zeros(B, dtype=torch.int64,
                                                                 device="cuda"))
    out = swa.swa_attn_decode_ring(to_dev(np.ascontiguousarray(q[:, :, N - 1])), rk, rv,
                                   torch.full((B,), N - 1, dtype=torch.int64, device="cuda"), 0.09)
    assert_close(to_f64(out), full[:, :, N - 1], what="decode==row")


def test_decode_workspace_reuse_and_exact_size(swa):
    B, H, Hkv, d, W = 2, 8, 2, 64, 512
    need = swa.swa_decode_workspace_bytes(B, H, Hkv, d, W)
    ws = torch.full((need,), 255, dtype=torch.uint8, device="cuda")  # garbage contents
    q = si.normal_bf16(3, 1, (B, H, d))
    rk = si.normal_bf16(3, 4, (B, Hkv, W, d))
    rv = si.normal_bf16(3, 5, (B, Hkv, W, d))
    a, _ = _run(swa, q, rk, rv, [600, 20], 0.125, workspace=ws)
    b, _ = _run(swa, q, rk, rv, [600, 20], 0.125, workspace=ws)
    assert np.array_equal(a, b)
    ref = oracle.swa_decode(q, rk, rv, [600, 20], W, 0.125)
    assert_close(a, ref)


@pytest.mark.parametrize("B,H,Hkv,d,W,S,pos", [
    (4, 32, 8, 128, 256, 4, [1000, 255, 258, 3]),       # sinks outside, none, some, partial ring
    (6, 4, 4, 64, 100, 16, [0, 5, 99, 100, 115, 5000]),  # G = 1, sinks entering the window
    (2, 16, 2, 128, 4096, 128, [4096 + 200, 70000]),    # G = 8, a full sink tile
    (1, 4, 2, 64, 1, 2, [9]),                           # W = 1: the query's own key plus two sinks
])
def test_decode_sink_full(swa, B, H, Hkv, d, W, S, pos):
    """Ring decode plus sinks (taxonomy page section 3.2) against the oracle.

    Compared with assert_close_bf16out: rows with W = 1 average three values.
    """
    seed = 900 + W + S
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, d))
    rk = si.normal_bf16(seed, si.STREAM["k_ring"], (B, Hkv, W, d))
    rv = si.normal_bf16(seed, si.STREAM["v_ring"], (B, Hkv, W, d))
    sk = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, S, d))
    sv = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, S, d))
    scale = 1.0 / math.sqrt(d)
    out, lse = swa.swa_attn_decode_ring(to_dev(q), to_dev(rk), to_dev(rv),
                                        torch.tensor(pos, dtype=torch.int64, device="cuda"),
                                        scale, return_lse=True, k_sink=to_dev(sk),
                                        v_sink=to_dev(sv))
    assert swa.swa_get_device_status() == 0
    ref, ref_lse = oracle.swa_decode_sink(q, rk, rv, sk, sv, pos, W, scale, with_lse=True)
    assert_close_bf16out(to_f64(out), ref, what="decode with sinks")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3


def test_decode_sink_workload_all_rows(swa):
    """The benchmarked decode with 4 sinks: every (b, h) row."""
    from swa_inputs.workloads import sink_inputs

    w = WORKLOADS["decode_ring_sink"]
    q, rk, rv, pos = decode_inputs(w)
    sk, sv = sink_inputs(w)
    out = swa.swa_attn_decode_ring(to_dev(q), to_dev(rk), to_dev(rv),
                                   torch.tensor(pos, dtype=torch.int64, device="cuda"), w.scale,
                                   k_sink=to_dev(sk), v_sink=to_dev(sv))
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_decode_sink(q, rk, rv, sk, sv, pos, w.W, w.scale)
    assert_close_bf16out(to_f64(out), ref, what="decode sink workload")


def test_decode_shift_by_window_is_identical(swa):
    """pos and pos + W see the same slots at the same relative positions."""
    B, H, Hkv, d, W = 4, 16, 4, 128, 1024
    pos = [5000, 1023, 77777, 2048]
    q = si.normal_bf16(61, si.STREAM["q"], (B, H, d))
    rk = si.normal_bf16(61, si.STREAM["k_ring"], (B, Hkv, W, d))
    rv = si.normal_bf16(61, si.STREAM["v_ring"], (B, Hkv, W, d))
    a, la = _run(swa, q, rk, rv, pos, 0.09)
    b, lb = _run(swa, q, rk, rv, [p + W for p in pos], 0.09)
    assert np.array_equal(a, b) and np.array_equal(la, lb)
