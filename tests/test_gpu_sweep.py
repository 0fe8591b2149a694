"""A seeded random sweep over small shapes of every path, against the oracle.

Each case draws B, the head layout (G = H / Hkv in {1, 2, 3, 4, 8}), d, the
window (from 1 to past the sequence), lengths that are not multiples of the
128-row tile, chunk starts on either side of the ring's wrap and sink counts,
so that edge combinations no hand-picked case covers are exercised.  Prefill
and packed rows that average at least 16 keys are held to the plain bar
(max-abs 1e-2, mean-abs 1e-3); rows of fewer keys, and the chunk and decode
cases, to the bf16-output bound (the 1e-2 bar plus 2^-8 of each value).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from tests._util import assert_close_bf16out, assert_close_by_keys, to_dev, to_f64

pytestmark = pytest.mark.gpu

N_CASES = 32


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _heads(rng):
    G = int(rng.choice([1, 2, 3, 4, 8]))
    Hkv = int(rng.integers(1, 3))
    return G * Hkv, Hkv


def _case(seed):
    rng = np.random.default_rng(seed)
    H, Hkv = _heads(rng)
    d = int(rng.choice([64, 128]))
    return rng, H, Hkv, d


@pytest.mark.parametrize("case", range(N_CASES))
def test_sweep_prefill(swa, case):
    rng, H, Hkv, d = _case(1000 + case)
    B = int(rng.integers(1, 3))
    N = int(rng.integers(1, 700))
    W = int(rng.choice([1, 2, int(rng.integers(3, 300)), N, N + 50]))
    S = int(rng.choice([0, 0, 1, 4]))
    q = si.normal_bf16(case, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(case, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(case, si.STREAM["v"], (B, Hkv, N, d))
    scale = 1.0 / math.sqrt(d)
    out = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, scale, n_sink=S)
    assert swa.swa_get_device_status() == 0
    got = to_f64(out)
    for b in range(B):
        tm = lambda x: np.ascontiguousarray(x[b].transpose(1, 0, 2))
        ref = oracle.swa_varlen(tm(q), tm(k), tm(v), [0, N], W, scale, n_sink=S)
        keys = np.minimum(np.arange(N) + 1, W)[:, None]  # [rows, 1]: per token, every head
        assert_close_by_keys(got[b].transpose(1, 0, 2), ref, keys,
                             what=f"prefill B{B} H{H}/{Hkv} N{N} d{d} W{W} S{S}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_sweep_chunk(swa, case):
    rng, H, Hkv, d = _case(2000 + case)
    B = int(rng.integers(1, 4))
    Tq = int(rng.integers(1, 300))
    W = int(rng.integers(1, 400))
    starts = [int(rng.choice([0, int(rng.integers(1, W + 1)), int(rng.integers(W, 5 * W + 2))]))
              for _ in range(B)]
    S = int(rng.choice([0, 0, 2]))
    if S:
        starts = [max(s, S) for s in starts]
    q = si.normal_bf16(case, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(case, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(case, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk = si.normal_bf16(case, si.STREAM["k_ring"], (B, Hkv, W, d))
    rv = si.normal_bf16(case, si.STREAM["v_ring"], (B, Hkv, W, d))
    scale = 1.0 / math.sqrt(d)
    tqs = torch.tensor(starts, dtype=torch.int64, device="cuda")
    kw = {}
    if S:
        sk = si.normal_bf16(case, si.STREAM["k_sink"], (B, Hkv, S, d))
        sv = si.normal_bf16(case, si.STREAM["v_sink"], (B, Hkv, S, d))
        kw = {"k_sink": to_dev(sk), "v_sink": to_dev(sv)}
    trk, trv = to_dev(rk), to_dev(rv)
    out = swa.swa_attn_chunk_ring(to_dev(q), to_dev(kn), to_dev(vn), trk, trv, tqs, scale,
                                  update_ring=True, **kw)
    assert swa.swa_get_device_status() == 0
    what = f"chunk B{B} H{H}/{Hkv} Tq{Tq} d{d} W{W} starts{starts} S{S}"
    if S:
        ref = oracle.swa_chunk_sink(q, kn, vn, rk, rv, sk, sv, starts, W, scale)
    else:
        ref = oracle.swa_chunk(q, kn, vn, rk, rv, starts, W, scale)
    assert_close_bf16out(to_f64(out), ref, what=what)
    from tests._util import to_host_bits

    erk, erv = oracle.ring_update(kn, vn, rk, rv, starts, W)
    assert np.array_equal(to_host_bits(trk), erk) and np.array_equal(to_host_bits(trv), erv)


@pytest.mark.parametrize("case", range(N_CASES))
def test_sweep_decode(swa, case):
    rng, H, Hkv, d = _case(3000 + case)
    if H // Hkv not in (1, 2, 4, 8):
        H = Hkv * 2
    B = int(rng.integers(1, 9))
    W = int(rng.integers(1, 3000))
    pos = [int(rng.integers(0, 4 * W + 10)) for _ in range(B)]
    S = int(rng.choice([0, 0, 3]))
    q = si.normal_bf16(case, si.STREAM["q"], (B, H, d))
    rk = si.normal_bf16(case, si.STREAM["k_ring"], (B, Hkv, W, d))
    rv = si.normal_bf16(case, si.STREAM["v_ring"], (B, Hkv, W, d))
    scale = 1.0 / math.sqrt(d)
    kw = {}
    if S:
        sk = si.normal_bf16(case, si.STREAM["k_sink"], (B, Hkv, S, d))
        sv = si.normal_bf16(case, si.STREAM["v_sink"], (B, Hkv, S, d))
        kw = {"k_sink": to_dev(sk), "v_sink": to_dev(sv)}
    out = swa.swa_attn_decode_ring(to_dev(q), to_dev(rk), to_dev(rv),
                                   torch.tensor(pos, dtype=torch.int64, device="cuda"), scale,
                                   **kw)
    assert swa.swa_get_device_status() == 0
    if S:
        ref = oracle.swa_decode_sink(q, rk, rv, sk, sv, pos, W, scale)
    else:
        ref = oracle.swa_decode(q, rk, rv, pos, W, scale)
    assert_close_bf16out(to_f64(out), ref, what=f"decode B{B} H{H}/{Hkv} d{d} W{W} S{S}")


@pytest.mark.parametrize("case", range(N_CASES))
def test_sweep_varlen(swa, case):
    rng, H, Hkv, d = _case(4000 + case)
    n_seq = int(rng.integers(1, 6))
    lens = [int(rng.choice([0, 1, int(rng.integers(2, 400))])) for _ in range(n_seq)]
    if sum(lens) == 0:
        lens[0] = 5
    W = int(rng.integers(1, 500))
    S = int(rng.choice([0, 0, 4]))
    total = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    q = si.normal_bf16(case, si.STREAM["q"], (total, H, d))
    k = si.normal_bf16(case, si.STREAM["k"], (total, Hkv, d))
    v = si.normal_bf16(case, si.STREAM["v"], (total, Hkv, d))
    scale = 1.0 / math.sqrt(d)
    out = swa.swa_attn_varlen(to_dev(q), to_dev(k), to_dev(v),
                              torch.tensor(cu, dtype=torch.int64, device="cuda"), max(lens), W,
                              scale, n_sink=S)
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_varlen(q, k, v, cu, W, scale, n_sink=S)
    pos = np.concatenate([np.arange(n) for n in lens])  # position of each token in its sequence
    keys = np.minimum(pos + 1, W)[:, None]
    assert_close_by_keys(to_f64(out), ref, keys, what=f"varlen lens{lens} H{H}/{Hkv} d{d} W{W} S{S}")


@pytest.mark.parametrize("case", range(16))
def test_sweep_backward(swa, case):
    """Gradients of random small shapes, each tensor bounded by its own scale
    (max-abs <= 8u max|ref|, mean-abs <= 2u mean|ref|, u = 2^-8)."""
    rng, H, Hkv, d = _case(5000 + case)
    B = int(rng.integers(1, 3))
    N = int(rng.integers(1, 600))
    W = int(rng.choice([1, int(rng.integers(2, 300)), N + 10]))
    q = si.normal_bf16(case, si.STREAM["q"], (B, H, N, d))
    k = si.normal_bf16(case, si.STREAM["k"], (B, Hkv, N, d))
    v = si.normal_bf16(case, si.STREAM["v"], (B, Hkv, N, d))
    g = si.normal_bf16(case, si.STREAM["extra"], (B, H, N, d))
    scale = 1.0 / math.sqrt(d)
    tq, tk, tv = to_dev(q), to_dev(k), to_dev(v)
    out, lse = swa.swa_attn_fwd(tq, tk, tv, W, scale, return_lse=True)
    grads = swa.swa_attn_bwd(tq, tk, tv, out, to_dev(g), lse, W, scale)
    assert swa.swa_get_device_status() == 0
    u = 2.0 ** -8
    for name, got, ref in zip(("dq", "dk", "dv"), grads, oracle.swa_backward(q, k, v, g, W, scale)):
        got = to_f64(got)
        err = np.abs(got - ref)
        what = f"backward {name} B{B} H{H}/{Hkv} N{N} d{d} W{W}"
        assert np.all(np.isfinite(got)), what
        if np.abs(ref).max() == 0:  # W = 1 or a single position: exactly 0 in the oracle
            assert err.max() < 1e-4, what
            continue
        assert err.max() <= 8 * u * np.abs(ref).max(), f"{what}: max-abs {err.max():.3e}"
        assert err.mean() <= 2 * u * np.abs(ref).mean(), f"{what}: mean-abs {err.mean():.3e}"
