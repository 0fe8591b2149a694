"""swa_attn_bwd (gradients of the windowed prefill) against the fp64 oracle.

The oracle differentiates sum(out * dout) exactly from the bf16 inputs; the
kernels round P and dS to bf16 for the tensor-core products (on the packed
layout the dK/dV kernel also forms dS from the rounded P) and write bf16
gradients.  Each of those roundings moves a value by at most u = 2^-8 of it,
so an entry's error is a few u times the size of the terms it sums.  The test
bounds each gradient tensor by its own scale: max-abs error <= 8u * max|ref|
and mean-abs error <= 2u * mean|ref|, and its relative RMS error (the error's
norm over the reference's) by 1e-2, about 2.5u: independent roundings of
relative size u add up in quadrature, not in the worst case.
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
    # the quadrature argument needs many entries; a gradient of a few rows
    # (a one- or two-token sequence) is held to the element bounds only
    norm = float(np.linalg.norm(ref))
    if ref.size >= 4096 and norm > 0:
        rel = float(np.linalg.norm(got - ref)) / norm
        assert rel <= 1e-2, f"{name}: relative RMS error {rel:.3e}"


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


# ---------------------------------------------------------------------------------------------
# Packed sequences (per-sequence windows) and attention sinks: the gradients of
# swa_attn_varlen / swa_attn_fwd_sink against oracle.swa_varlen_backward, which
# finite differences and torch autograd pin (tests/test_oracle_pins.py).

def _varlen_inputs(seed, lens, H, Hkv, d, total_extra=0):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    total = int(cu[-1]) + total_extra
    q = si.normal_bf16(seed, si.STREAM["q"], (total, H, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (total, Hkv, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (total, Hkv, d))
    g = si.normal_bf16(seed, si.STREAM["extra"], (total, H, d))
    return q, k, v, g, cu


@pytest.mark.parametrize("lens,H,Hkv,d,W,S", [
    ([300, 1, 129, 0, 640], 4, 2, 128, 100, 0),      # ragged, a one-token and an empty sequence
    ([300, 1, 129, 0, 640], 4, 2, 128, 100, 4),      # the same with four sinks
    ([257, 512, 77], 3, 1, 64, 64, 16),              # G = 3, d = 64, sinks across a tile
    ([1000, 130], 8, 2, 128, 129, 128),              # a full key tile of sinks
    ([700, 384, 1025], 8, 8, 128, 4096, 4),          # window beyond every sequence: causal
    ([200, 333], 2, 2, 128, 1, 2),                   # W = 1 plus sinks
    ([2500, 4100], 4, 2, 128, 1024, 4),              # sink key tile read by 33 query tiles
])
def test_varlen_backward(swa, lens, H, Hkv, d, W, S):
    seed = 500 + sum(lens) + W + S
    q, k, v, g, cu = _varlen_inputs(seed, lens, H, Hkv, d)
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    max_len = max(lens)
    out, lse = swa.swa_attn_varlen(tq, tk, tv, tcu, max_len, W, scale, n_sink=S, return_lse=True)
    dq, dk, dv = swa.swa_attn_varlen_bwd(tq, tk, tv, tcu, max_len, out, tg, lse, W, scale,
                                         n_sink=S)
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_varlen_backward(q, k, v, g, cu, W, scale, n_sink=S)
    for name, a, b in zip(("dq", "dk", "dv"), (to_f64(dq), to_f64(dk), to_f64(dv)), ref):
        if W == 1 and name != "dv" and S == 0:
            assert np.max(np.abs(a)) < 1e-4
            continue
        _check(name, a, b)


def test_varlen_backward_leaves_rows_outside_sequences(swa):
    """Tokens after the last sequence: their gradient rows keep what the caller put there."""
    lens, H, Hkv, d, W = [130, 200], 4, 2, 128, 64
    q, k, v, g, cu = _varlen_inputs(61, lens, H, Hkv, d, total_extra=50)
    total = q.shape[0]
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    out, lse = swa.swa_attn_varlen(tq, tk, tv, tcu, 200, W, 0.1, n_sink=2, return_lse=True)
    fill = lambda t: torch.full_like(t, 7.0)  # noqa: E731
    dq, dk, dv = swa.swa_attn_varlen_bwd(tq, tk, tv, tcu, 200, out, tg, lse, W, 0.1, n_sink=2,
                                         dq=fill(tq), dk=fill(tk), dv=fill(tv))
    assert swa.swa_get_device_status() == 0
    n = int(cu[-1])
    for t in (dq, dk, dv):
        assert bool(torch.all(t[n:] == 7.0))
    ref = oracle.swa_varlen_backward(q[:n], k[:n], v[:n], g[:n], cu, W, 0.1, n_sink=2)
    for name, a, b in zip(("dq", "dk", "dv"), (dq[:n], dk[:n], dv[:n]), ref):
        _check(name, to_f64(a), b)
    del total


def test_varlen_backward_sequences_do_not_mix(swa):
    """Changing one sequence's tokens leaves every other sequence's gradients bit-identical."""
    lens, H, Hkv, d, W = [256, 300, 129], 4, 2, 128, 200
    q, k, v, g, cu = _varlen_inputs(62, lens, H, Hkv, d)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")

    def grads(qq, kk, vv, gg):
        tq, tk, tv, tg = to_dev(qq), to_dev(kk), to_dev(vv), to_dev(gg)
        out, lse = swa.swa_attn_varlen(tq, tk, tv, tcu, 300, W, 0.1, n_sink=4, return_lse=True)
        return swa.swa_attn_varlen_bwd(tq, tk, tv, tcu, 300, out, tg, lse, W, 0.1, n_sink=4)

    a = grads(q, k, v, g)
    k2, v2 = k.copy(), v.copy()
    k2[256:556] = si.normal_bf16(63, 2, k2[256:556].shape)
    v2[256:556] = si.normal_bf16(63, 3, v2[256:556].shape)
    b = grads(q, k2, v2, g)
    for x, y in zip(a, b):
        assert torch.equal(x[:256], y[:256]) and torch.equal(x[556:], y[556:])


@pytest.mark.parametrize("B,H,Hkv,N,d,W,S", [
    (1, 4, 2, 300, 128, 100, 4),
    (2, 2, 1, 700, 64, 129, 128),
])
def test_backward_with_sinks(swa, B, H, Hkv, N, d, W, S):
    """swa_attn_bwd_sink on the [B, H, N, d] layout: each batch entry is one sequence."""
    seed = 70 + N + S
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(seed, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(seed, si.STREAM["v"], (B, Hkv, N, d))
    g = si.normal_bf16(seed, si.STREAM["extra"], (B, H, N, d))
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = swa.swa_attn_fwd(tq, tk, tv, W, scale, return_lse=True, n_sink=S)
    dq, dk, dv = swa.swa_attn_bwd(tq, tk, tv, out, tg, lse, W, scale, n_sink=S)
    assert swa.swa_get_device_status() == 0
    got = (to_f64(dq), to_f64(dk), to_f64(dv))
    tok = lambda x: np.ascontiguousarray(x.transpose(0, 2, 1, 3).reshape(-1, x.shape[1], d))  # noqa: E731
    cu = np.arange(B + 1, dtype=np.int64) * N
    ref = oracle.swa_varlen_backward(tok(q), tok(k), tok(v), tok(g), cu, W, scale, n_sink=S)
    for name, a, b in zip(("dq", "dk", "dv"), got, ref):
        _check(name, tok(a), b)


def test_varlen_backward_workload_sampled(swa):
    """The benchmarked packed batch with sinks (16 sequences of 256..16384 tokens): every
    gradient row of the sequences of at most 4096 tokens (the oracle's cost grows with
    length times window; the longer ones run the same code on more tiles)."""
    from swa_inputs.workloads import WORKLOADS, seq_lens, varlen_inputs

    w = WORKLOADS["varlen_backward"]
    q, k, v, cu = varlen_inputs(w)
    g = si.normal_bf16(w.seed, si.STREAM["extra"], q.shape)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    lens = seq_lens(w)
    max_len = int(max(lens))
    out, lse = swa.swa_attn_varlen(tq, tk, tv, tcu, max_len, w.W, w.scale, n_sink=w.n_sink,
                                   return_lse=True)
    dq, dk, dv = swa.swa_attn_varlen_bwd(tq, tk, tv, tcu, max_len, out, tg, lse, w.W, w.scale,
                                         n_sink=w.n_sink)
    assert swa.swa_get_device_status() == 0
    short = [s for s in range(len(lens)) if lens[s] <= 4096]
    assert short
    for s in short:
        a, e = int(cu[s]), int(cu[s + 1])
        ref = oracle.swa_varlen_backward(q[a:e], k[a:e], v[a:e], g[a:e], np.array([0, e - a]),
                                         w.W, w.scale, n_sink=w.n_sink)
        for name, x, y in zip(("dq", "dk", "dv"), (dq[a:e], dk[a:e], dv[a:e]), ref):
            _check(f"{name} seq {s} ({e - a} tokens)", to_f64(x), y)


def test_varlen_backward_workload_long_sequence_one_group(swa):
    """The benchmarked packed batch with sinks: every gradient element of its shortest
    sequence longer than W + 1024 (5284 tokens: a thousand rows whose window no longer
    reaches the 4 sinks) for key/value head 0's group (dq of its query heads, dk and dv
    of the key head), which depend on that group and that sequence alone."""
    from swa_inputs.workloads import WORKLOADS, seq_lens, varlen_inputs

    w = WORKLOADS["varlen_backward"]
    q, k, v, cu = varlen_inputs(w)
    g = si.normal_bf16(w.seed, si.STREAM["extra"], q.shape)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    lens = seq_lens(w)
    max_len = int(max(lens))
    out, lse = swa.swa_attn_varlen(tq, tk, tv, tcu, max_len, w.W, w.scale, n_sink=w.n_sink,
                                   return_lse=True)
    dq, dk, dv = swa.swa_attn_varlen_bwd(tq, tk, tv, tcu, max_len, out, tg, lse, w.W, w.scale,
                                         n_sink=w.n_sink)
    assert swa.swa_get_device_status() == 0
    longer = [i for i in range(len(lens)) if lens[i] > w.W + 1024]
    s = min(longer, key=lambda i: lens[i])
    a, e = int(cu[s]), int(cu[s + 1])
    G = w.H // w.Hkv
    sl = lambda x, n: np.ascontiguousarray(x[a:e, :n])  # noqa: E731
    ref = oracle.swa_varlen_backward(sl(q, G), sl(k, 1), sl(v, 1), sl(g, G),
                                     np.array([0, e - a]), w.W, w.scale, n_sink=w.n_sink)
    for name, x, y in zip(("dq", "dk", "dv"),
                          (dq[a:e, :G], dk[a:e, :1], dv[a:e, :1]), ref):
        _check(f"{name} seq {s} ({e - a} tokens), group 0", to_f64(x), y)
