"""swa_attn_bwd (gradients of the windowed prefill) against the fp64 oracle.

The oracle differentiates sum(out * dout) exactly from the bf16 inputs; the
kernels round P and dS to bf16 for the tensor-core products and write bf16
gradients.  Each of those roundings moves a value by at most u = 2^-8 of it,
so an entry's error is a few u times the size of the terms it sums.  The test
bounds each gradient tensor by its own scale: max-abs error <= 8u * max|ref|
and mean-abs error <= 2u * mean|ref|.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from tests._util import to_dev, to_f64

pytestmark = pytest.mark.gpu

U = 2.0 ** -8


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _check(name, got, ref):
    err = np.abs(got - ref)
    mx, mn = float(err.max()), float(err.mean())
    assert np.all(np.isfinite(got)), f"{name}: non-finite"
    assert mx <= 8 * U * float(np.abs(ref).max()) and mn <= 2 * U * float(np.abs(ref).mean()), \
        f"{name}: max-abs {mx:.3e} (ref max {np.abs(ref).max():.3e}), mean-abs {mn:.3e} " \
        f"(ref mean {np.abs(ref).mean():.3e})"


def _run(swa, B, H, Hkv, N, d, W, seed):
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, N, d))
    g = si.normal_bf16(seed, si.STREAM["extra"], (B, H, N, d))
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = swa.swa_attn_fwd(tq, tk, tv, W, scale, return_lse=True)
    dq, dk, dv = swa.swa_attn_bwd(tq, tk, tv, out, tg, lse, W, scale)
    assert swa.swa_get_device_status() == 0
    rq, rk, rv = oracle.swa_backward(q, k, v, g, W, scale)
    return (to_f64(dq), to_f64(dk), to_f64(dv)), (rq, rk, rv)


@pytest.mark.parametrize("B,H,Hkv,N,d,W", [
    (1, 4, 2, 300, 128, 100),      # ragged tail, window across three key tiles
    (2, 3, 1, 257, 64, 64),        # G = 3, d = 64, one row past a tile
    (1, 8, 2, 512, 128, 1000),     # window covers everything: causal attention
    (1, 2, 2, 130, 128, 1),        # W = 1: dq = dk = 0 up to rounding
    (1, 8, 8, 640, 128, 256),      # G = 1, aligned tiles, full and partial tiles
    (1, 4, 1, 384, 64, 129),       # G = 4, window one past a tile
])
def test_backward_small(swa, B, H, Hkv, N, d, W):
    got, ref = _run(swa, B, H, Hkv, N, d, W, seed=40 + N + W)
    if W == 1:
        # exactly 0 in the oracle; here dS = P (dP - D) with dP (tensor cores) and
        # D (FMA) two fp32 dot products of the same 128 terms, equal up to rounding
        assert np.max(np.abs(got[0])) < 1e-4 and np.max(np.abs(got[1])) < 1e-4
        _check("dv", got[2], ref[2])
        return
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        _check(name, a, b)


def test_backward_medium(swa):
    """Many tiles per window, GQA 4: every gradient entry."""
    got, ref = _run(swa, 1, 8, 2, 4096, 128, 2048, seed=77)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        _check(name, a, b)


def test_backward_workspace_too_small(swa):
    from sliding_window_sparse_b200._native import SwaError

    B, H, Hkv, N, d = 1, 2, 2, 128, 64
    x = torch.zeros((B, H, N, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, H, N), dtype=torch.float32, device="cuda")
    with pytest.raises(SwaError):
        swa.swa_attn_bwd(x, x, x, x, x, lse, 16, workspace=torch.empty(16, dtype=torch.uint8,
                                                                      device="cuda"))
