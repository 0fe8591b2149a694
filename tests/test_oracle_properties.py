"""Properties of the oracle over randomly drawn small shapes (CPU, hypothesis).

The pins in test_oracle_pins.py check fixed cases; these draw the shapes,
windows, chunkings and positions at random (derandomized, so every run sees
the same examples) and check that the oracle's independent paths agree:

* the pair loop equals the dense score table with the window mask (M003
  note section 07's baseline; the difference convention of Chapter 10
  section 10.1);
* a prefill cut into chunks over a W-slot ring equals the one-pass prefill
  exactly (Chapter 10 section 10.2; the ring of the blog's section 3.2);
* decode at position p equals row p of the prefill;
* packed sequences equal separate prefills of each sequence (blog section
  5.2 tip 4: windows never cross a sequence boundary);
* the benchmark's closed-form pair count equals the enumeration, sinks
  included (taxonomy page section 3.2);
* with sinks, chunks over a ring and decode both equal the one-pass packed
  prefill with the same sinks.
"""

import os
import sys

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
import swa_inputs as si  # noqa: E402

SETTINGS = settings(max_examples=80, deadline=None, derandomize=True, database=None,
                    suppress_health_check=[HealthCheck.too_slow])


def _draw(seed, shape, stream):
    return si.normal_bf16(seed, si.STREAM[stream], shape)


def _qkv(seed, B, H, Hkv, N, d):
    return (_draw(seed, (B, H, N, d), "q"), _draw(seed, (B, Hkv, N, d), "k"),
            _draw(seed, (B, Hkv, N, d), "v"))


heads = st.sampled_from([(1, 1), (2, 1), (4, 2), (3, 3), (6, 2)])


@SETTINGS
@given(seed=st.integers(0, 10_000), hk=heads, N=st.integers(1, 40), W=st.integers(1, 50),
       d=st.sampled_from([4, 8, 16]))
def test_pair_loop_equals_dense_mask(seed, hk, N, W, d):
    H, Hkv = hk
    q, k, v = _qkv(seed, 1, H, Hkv, N, d)
    a = oracle.swa_forward(q, k, v, W, 0.4)
    b = oracle.dense_masked(q, k, v, W, 0.4)
    assert np.max(np.abs(a - b)) < 1e-12


@SETTINGS
@given(seed=st.integers(0, 10_000), N=st.integers(2, 60), W=st.integers(1, 24),
       cuts=st.lists(st.integers(1, 59), max_size=5))
def test_chunked_over_ring_equals_one_pass(seed, N, W, cuts):
    B, H, Hkv, d = 1, 2, 1, 8
    q, k, v = _qkv(seed, B, H, Hkv, N, d)
    bounds = sorted({c for c in cuts if c < N} | {0, N})
    rk = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    rv = np.zeros_like(rk)
    outs = []
    for c0, c1 in zip(bounds[:-1], bounds[1:]):
        outs.append(oracle.swa_chunk(q[:, :, c0:c1], k[:, :, c0:c1], v[:, :, c0:c1], rk, rv,
                                     [c0], W, 0.5))
        rk, rv = oracle.ring_update(k[:, :, c0:c1], v[:, :, c0:c1], rk, rv, [c0], W)
    assert np.array_equal(np.concatenate(outs, axis=2), oracle.swa_forward(q, k, v, W, 0.5))


@SETTINGS
@given(seed=st.integers(0, 10_000), P=st.integers(0, 70), W=st.integers(1, 40))
def test_decode_equals_prefill_row(seed, P, W):
    B, H, Hkv, d = 1, 4, 2, 8
    q, k, v = _qkv(seed, B, H, Hkv, P + 1, d)
    rk = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    rv = np.zeros_like(rk)
    rk, rv = oracle.ring_update(k, v, rk, rv, [0], W)
    dec = oracle.swa_decode(np.ascontiguousarray(q[:, :, P]), rk, rv, [P], W, 0.3)
    assert np.array_equal(dec, oracle.swa_forward(q, k, v, W, 0.3)[:, :, P])


@SETTINGS
@given(seed=st.integers(0, 10_000), lens=st.lists(st.integers(1, 20), min_size=1, max_size=5),
       W=st.integers(1, 25), hk=heads)
def test_packed_sequences_equal_separate_prefills(seed, lens, W, hk):
    H, Hkv, d = hk[0], hk[1], 8
    total = sum(lens)
    q = _draw(seed, (total, H, d), "q")
    k = _draw(seed, (total, Hkv, d), "k")
    v = _draw(seed, (total, Hkv, d), "v")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    packed = oracle.swa_varlen(q, k, v, cu, W, 0.6)
    for s, n in enumerate(lens):
        a, b = int(cu[s]), int(cu[s + 1])
        one = oracle.swa_forward(q[a:b].transpose(1, 0, 2)[None], k[a:b].transpose(1, 0, 2)[None],
                                 v[a:b].transpose(1, 0, 2)[None], W, 0.6)
        assert np.array_equal(packed[a:b], one[0].transpose(1, 0, 2))


@SETTINGS
@given(N=st.integers(1, 120), W=st.integers(1, 130), S=st.integers(0, 10))
def test_closed_form_pairs_equal_enumeration(N, W, S):
    assert bench.sequence_pairs(N, W, S) == oracle.count_pairs_sink(N, W, S)


@SETTINGS
@given(seed=st.integers(0, 10_000), N=st.integers(2, 60), W=st.integers(1, 20),
       S=st.integers(1, 6), cuts=st.lists(st.integers(1, 59), max_size=4))
def test_chunked_with_sinks_equals_one_pass(seed, N, W, S, cuts):
    """Chunks over a ring plus sink rows equal the one-pass prefill with the same
    sinks (taxonomy page section 3.2 on Chapter 10 section 10.2)."""
    B, H, Hkv, d = 1, 2, 1, 8
    S = min(S, N)
    q, k, v = _qkv(seed, B, H, Hkv, N, d)
    tm = lambda x: np.ascontiguousarray(x[0].transpose(1, 0, 2))
    full = oracle.swa_varlen(tm(q), tm(k), tm(v), [0, N], W, 0.45, n_sink=S).transpose(1, 0, 2)
    sk = np.ascontiguousarray(k[:, :, :S])
    sv = np.ascontiguousarray(v[:, :, :S])
    rk = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    rv = np.zeros_like(rk)
    bounds = sorted({c for c in cuts if c < N} | {0, N})
    for a, e in zip(bounds[:-1], bounds[1:]):
        sl = (slice(None), slice(None), slice(a, e))
        qc, kc, vc = (np.ascontiguousarray(x[sl]) for x in (q, k, v))
        out = oracle.swa_chunk_sink(qc, kc, vc, rk, rv, sk, sv, [a], W, 0.45)
        assert np.array_equal(out[0], full[:, a:e])
        rk, rv = oracle.ring_update(kc, vc, rk, rv, [a], W)


@SETTINGS
@given(seed=st.integers(0, 10_000), P=st.integers(0, 60), W=st.integers(1, 30),
       S=st.integers(0, 6))
def test_decode_with_sinks_equals_prefill_row(seed, P, W, S):
    B, H, Hkv, d = 1, 4, 2, 8
    N = P + 1
    q, k, v = _qkv(seed, B, H, Hkv, N, d)
    rk = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    rv = np.zeros_like(rk)
    rk, rv = oracle.ring_update(k, v, rk, rv, [0], W)
    sk = np.zeros((B, Hkv, S, d), dtype=np.uint16)
    sv = np.zeros_like(sk)
    n_s = min(S, N)
    sk[:, :, :n_s] = k[:, :, :n_s]
    sv[:, :, :n_s] = v[:, :, :n_s]
    dec = oracle.swa_decode_sink(np.ascontiguousarray(q[:, :, P]), rk, rv, sk, sv, [P], W, 0.4)
    tm = lambda x: np.ascontiguousarray(x[0].transpose(1, 0, 2))
    full = oracle.swa_varlen(tm(q), tm(k), tm(v), [0, N], W, 0.4, n_sink=S)
    assert np.array_equal(dec[0], full[P])
