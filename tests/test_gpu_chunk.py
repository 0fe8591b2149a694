"""swa_attn_chunk_ring (chunked prefill on a ring cache) and swa_ring_write vs the oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from swa_inputs.workloads import WORKLOADS, chunk_inputs
from tests._util import assert_close, sample_rows, to_dev, to_f64, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _ring_from_history(seed, B, Hkv, W, d, q_starts):
    """Ring contents after writing positions 0..q_start-1 (random rows per position)."""
    rk = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    rv = np.zeros((B, Hkv, W, d), dtype=np.uint16)
    for b, qs in enumerate(q_starts):
        if qs == 0:
            continue
        n = min(qs, W)
        kk = si.normal_bf16(seed + b, si.STREAM["k_ring"], (1, Hkv, n, d))
        vv = si.normal_bf16(seed + b, si.STREAM["v_ring"], (1, Hkv, n, d))
        k1, v1 = oracle.ring_update(kk, vv, rk[b:b + 1], rv[b:b + 1], [qs - n], W)
        rk[b:b + 1], rv[b:b + 1] = k1, v1
    return rk, rv


def _run(swa, q, kn, vn, rk, rv, qs, scale, update=False):
    tq, tkn, tvn, trk, trv = (to_dev(x) for x in (q, kn, vn, rk, rv))
    tqs = torch.tensor(qs, dtype=torch.int64, device="cuda")
    out, lse = swa.swa_attn_chunk_ring(tq, tkn, tvn, trk, trv, tqs, scale, update_ring=update,
                                       return_lse=True)
    assert swa.swa_get_device_status() == 0
    return out, lse, trk, trv


@pytest.mark.parametrize("B,H,Hkv,Tq,d,W,starts", [
    (2, 4, 2, 64, 128, 256, [512, 600]),          # aligned and unaligned ring
    (2, 4, 4, 200, 64, 128, [1000, 77]),          # chunk longer than the window
    (3, 2, 1, 130, 128, 300, [0, 5, 301]),        # empty ring, partly filled, ragged tiles
    (1, 8, 2, 1, 128, 64, [900]),                 # one-token chunk
    (1, 4, 2, 384, 128, 512, [12288 + 37]),       # unaligned large start
])
def test_small_chunks_full_tensor(swa, B, H, Hkv, Tq, d, W, starts):
    seed = 300 + Tq + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    scale = 1.0 / math.sqrt(d)
    out, lse, trk, trv = _run(swa, q, kn, vn, rk, rv, starts, scale, update=True)
    ref, ref_lse = oracle.swa_chunk(q, kn, vn, rk, rv, starts, W, scale, with_lse=True)
    assert_close(to_f64(out), ref, what="chunk")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3
    erk, erv = oracle.ring_update(kn, vn, rk, rv, starts, W)
    assert np.array_equal(to_host_bits(trk), erk)
    assert np.array_equal(to_host_bits(trv), erv)


def test_chunk_workload_sampled_rows(swa):
    w = WORKLOADS["chunk_ring"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    out, _, _, _ = _run(swa, q, kn, vn, rk, rv, list(qs), w.scale)
    edges = [0, 1, 127, 128, 255, 256, 383, 384, 510, 511]
    rows = sample_rows(w.B, w.H, w.Tq, 200, seed=11, extra=edges)
    ref = oracle.swa_chunk(q, kn, vn, rk, rv, qs, w.W, w.scale, rows=rows)
    got = to_f64(out)[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_close(got, ref, what="chunk_ring workload")
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-2


@pytest.mark.parametrize("needle_rel", [50, -1, 10])
def test_chunk_needle_unaligned_ring(swa, needle_rel):
    """A dominating key in the ring (past the wrap of an unaligned ring) or in the
    chunk: query t sees it iff its position is in [q_start + t - W + 1, q_start + t]."""
    W, Tq, d = 512, 256, 128
    q_start = 4096 + 37
    # needle_rel > 0 counts from the oldest ring position, < 0 from the newest,
    # and 10 puts it in the chunk
    p_star = q_start - W + needle_rel if needle_rel != 10 else q_start + 10
    if needle_rel < 0:
        p_star = q_start + needle_rel
    u = np.zeros(d, dtype=np.float32)
    u[:8] = 1.0
    qf = np.tile(u, (1, 1, Tq, 1))
    knf = si.bf16_bits_to_f32(si.normal_bf16(6, si.STREAM["k_new"], (1, 1, Tq, d))) * 0.1
    rkf = si.bf16_bits_to_f32(si.normal_bf16(6, si.STREAM["k_ring"], (1, 1, W, d))) * 0.1
    needle = 8.0 * u / np.linalg.norm(u) * math.sqrt(d)
    if p_star >= q_start:
        knf[0, 0, p_star - q_start] = needle
    else:
        rkf[0, 0, p_star % W] = needle  # slot = position mod W
    q, kn, rk = (si.f32_to_bf16_bits(x.astype(np.float32)) for x in (qf, knf, rkf))
    vn = si.normal_bf16(6, si.STREAM["v_new"], (1, 1, Tq, d))
    rv = si.normal_bf16(6, si.STREAM["v_ring"], (1, 1, W, d))
    scale = 1.0 / math.sqrt(d)
    out, _, _, _ = _run(swa, q, kn, vn, rk, rv, [q_start], scale)
    got = to_f64(out)[0, 0]
    ref = oracle.swa_chunk(q, kn, vn, rk, rv, [q_start], W, scale)[0, 0]
    assert_close(got, ref, what="chunk needle")
    vsrc = vn[0, 0, p_star - q_start] if p_star >= q_start else rv[0, 0, p_star % W]
    vneedle = si.bf16_bits_to_f32(vsrc).astype(np.float64)
    for t in range(Tq):
        sees = q_start + t - W + 1 <= p_star <= q_start + t
        close = np.max(np.abs(got[t] - vneedle)) < 0.05
        assert close == sees, f"query {t}: sees needle {sees}, output matches {close}"


def test_chunk_shift_by_window_is_identical(swa):
    """The same ring contents at q_start and q_start + W hold the same relative
    positions (slot = position mod W), so the outputs are bit-identical."""
    B, H, Hkv, Tq, d, W = 2, 8, 2, 200, 128, 384
    starts = [5000 + 77, 1000]
    seed = 55
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    a, la, _, _ = _run(swa, q, kn, vn, rk, rv, starts, 0.1)
    b, lb, _, _ = _run(swa, q, kn, vn, rk, rv, [s + W for s in starts], 0.1)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_chunked_equals_full_prefill(swa):
    """Chapter 10 section 10.5: full forward == chunks [0:2], [2:5], [5:7] through the ring
    (7 tokens, W = 3), and the same on a larger case with ragged chunks."""
    for N, W, chunks in [(7, 3, [(0, 2), (2, 5), (5, 7)]),
                         (700, 200, [(0, 100), (100, 101), (101, 450), (450, 700)])]:
        B, H, Hkv, d = 1, 4, 2, 128
        q = si.normal_bf16(9, si.STREAM["q"], (B, H, N, d))
        k = si.normal_bf16(9, si.STREAM["k"], (B, Hkv, N, d))
        v = si.normal_bf16(9, si.STREAM["v"], (B, Hkv, N, d))
        full = to_f64(swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, 0.1))
        rk = torch.zeros((B, Hkv, W, d), dtype=torch.bfloat16, device="cuda")
        rv = torch.zeros_like(rk)
        parts = []
        for c0, c1 in chunks:
            qs = torch.tensor([c0], dtype=torch.int64, device="cuda")
            o = swa.swa_attn_chunk_ring(to_dev(np.ascontiguousarray(q[:, :, c0:c1])),
                                        to_dev(np.ascontiguousarray(k[:, :, c0:c1])),
                                        to_dev(np.ascontiguousarray(v[:, :, c0:c1])),
                                        rk, rv, qs, 0.1, update_ring=True)
            parts.append(to_f64(o))
        chunked = np.concatenate(parts, axis=2)
        assert_close(chunked, full, what=f"chunked N{N}")
        ref = oracle.swa_forward(q, k, v, W, 0.1)
        assert_close(chunked, ref, what="chunked vs oracle")


def test_ring_write_bit_exact(swa):
    B, Hkv, T, d, W = 3, 2, 70, 64, 32
    kn = si.normal_bf16(1, 6, (B, Hkv, T, d))
    vn = si.normal_bf16(1, 7, (B, Hkv, T, d))
    rk = si.normal_bf16(1, 4, (B, Hkv, W, d))
    rv = si.normal_bf16(1, 5, (B, Hkv, W, d))
    starts = [0, 31, 1000]
    trk, trv = to_dev(rk), to_dev(rv)
    swa.swa_ring_write(to_dev(kn), to_dev(vn), trk, trv,
                       torch.tensor(starts, dtype=torch.int64, device="cuda"))
    erk, erv = oracle.ring_update(kn, vn, rk, rv, starts, W)
    assert np.array_equal(to_host_bits(trk), erk)
    assert np.array_equal(to_host_bits(trv), erv)


def test_negative_start_reports_device_error(swa):
    B, H, Hkv, Tq, d, W = 1, 2, 2, 16, 64, 32
    z = torch.zeros((B, H, Tq, d), dtype=torch.bfloat16, device="cuda")
    zk = torch.zeros((B, Hkv, Tq, d), dtype=torch.bfloat16, device="cuda")
    rk = torch.zeros((B, Hkv, W, d), dtype=torch.bfloat16, device="cuda")
    qs = torch.tensor([-1], dtype=torch.int64, device="cuda")
    swa.swa_attn_chunk_ring(z, zk, zk, rk, rk.clone(), qs, 0.1)
    assert swa.swa_get_device_status() == 6


def _run_ragged(swa, q, kn, vn, rk, rv, qs, lens, scale, update=False, fill=7.0):
    tq, tkn, tvn, trk, trv = (to_dev(x) for x in (q, kn, vn, rk, rv))
    tqs = torch.tensor(qs, dtype=torch.int64, device="cuda")
    tl = torch.tensor(lens, dtype=torch.int64, device="cuda")
    out = torch.full_like(tq, fill)
    lse = torch.full(tq.shape[:3], fill, dtype=torch.float32, device="cuda")
    swa.swa_attn_chunk_ring_ragged(tq, tkn, tvn, trk, trv, tqs, tl, scale, update_ring=update,
                                   out=out, lse=lse, return_lse=True)
    assert swa.swa_get_device_status() == 0
    return out, lse, trk, trv


@pytest.mark.parametrize("B,H,Hkv,Tq,d,W,starts,lens", [
    # full, one token, ends one row past a tile, empty
    (4, 4, 2, 300, 128, 256, [512, 40, 0, 700], [300, 1, 129, 0]),
    # odd group size (q-tile pairs), chunk longer than the window, mid-tile ends
    (3, 6, 2, 256, 64, 128, [1000, 3, 129], [200, 256, 65]),
    # GQA 4:1 with even group (head pairs), lengths either side of a 128-row tile
    (3, 8, 2, 384, 128, 512, [12288 + 37, 0, 511], [127, 128, 383]),
])
def test_ragged_chunks_per_sequence(swa, B, H, Hkv, Tq, d, W, starts, lens):
    """Each sequence b equals a plain chunk call on its first lens[b] rows (Chapter 10 s10.2)."""
    seed = 900 + Tq + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    scale = 1.0 / math.sqrt(d)
    out, lse, trk, trv = _run_ragged(swa, q, kn, vn, rk, rv, starts, lens, scale, update=True)
    got, got_lse = to_f64(out), to_f64(lse)
    erk, erv = rk.copy(), rv.copy()
    for b, (qs, n) in enumerate(zip(starts, lens)):
        # padding rows stay as the caller left them
        assert np.all(got[b, :, n:] == 7.0)
        assert np.all(got_lse[b, :, n:] == 7.0)
        if n == 0:
            continue
        sl = (slice(b, b + 1), slice(None), slice(0, n))
        ref, ref_lse = oracle.swa_chunk(q[sl], kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [qs], W,
                                        scale, with_lse=True)
        assert_close(got[b:b + 1, :, :n], ref, what=f"ragged chunk b={b} len={n}")
        assert np.max(np.abs(got_lse[b:b + 1, :, :n] - ref_lse)) < 1e-3
        k1, v1 = oracle.ring_update(kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [qs], W)
        erk[b:b + 1], erv[b:b + 1] = k1, v1
    assert np.array_equal(to_host_bits(trk), erk)
    assert np.array_equal(to_host_bits(trv), erv)


def test_ragged_full_lengths_match_plain_call(swa):
    """chunk_len = Tq everywhere is bit-identical to swa_attn_chunk_ring."""
    B, H, Hkv, Tq, d, W = 2, 8, 2, 320, 128, 256
    starts = [4096 + 5, 300]
    seed = 77
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    scale = 1.0 / math.sqrt(d)
    o1, l1, _, _ = _run(swa, q, kn, vn, rk, rv, starts, scale)
    o2, l2, _, _ = _run_ragged(swa, q, kn, vn, rk, rv, starts, [Tq] * B, scale)
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)



def test_ragged_chunk_workload_sampled_rows(swa):
    """The benchmarked ragged chunk batch (1..512 valid rows per sequence), sampled rows."""
    from swa_inputs.workloads import seq_lens

    w = WORKLOADS["chunk_ring_ragged"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    lens = [int(n) for n in seq_lens(w)]
    out, _, _, _ = _run_ragged(swa, q, kn, vn, rk, rv, list(qs), lens, w.scale)
    got = to_f64(out)
    rng = np.random.default_rng(12)
    for b, n in enumerate(lens):
        ts = sorted(set(rng.integers(0, n, 40).tolist()) | {0, n - 1, min(127, n - 1)})
        rows = np.array([(0, int(rng.integers(w.H)), t) for t in ts], dtype=np.int64)
        sl = (slice(b, b + 1), slice(None), slice(0, n))
        ref = oracle.swa_chunk(q[sl], kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [int(qs[b])],
                               w.W, w.scale, rows=rows)
        assert_close(got[b, rows[:, 1], rows[:, 2]], ref, what=f"ragged chunk workload b={b}")
        assert np.all(got[b, :, n:] == 7.0)


@pytest.mark.parametrize("B,H,Hkv,Tq,d,W,S,starts", [
    (2, 8, 2, 200, 128, 256, 4, [5000 + 77, 300]),   # head pairs, sinks before the window
    (3, 6, 2, 130, 64, 100, 16, [1000, 77, 3]),      # query-tile pairs; a start below S
    (1, 4, 2, 64, 128, 512, 4, [10]),                # no query sees a sink: sink tile skipped
    (1, 2, 1, 300, 128, 128, 128, [4096]),           # a full tile of sinks
])
def test_chunk_with_sinks(swa, B, H, Hkv, Tq, d, W, S, starts):
    """Chunk over the ring plus sink rows (taxonomy page section 3.2) vs the oracle."""
    from tests._util import assert_close_bf16out

    seed = 1200 + Tq + W + S
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    sk = si.normal_bf16(seed, si.STREAM["k_sink"], (B, Hkv, S, d))
    sv = si.normal_bf16(seed, si.STREAM["v_sink"], (B, Hkv, S, d))
    for b, qs in enumerate(starts):  # sink positions inside the chunk: its own rows
        for j in range(qs, min(S, qs + Tq)):
            sk[b, :, j] = kn[b, :, j - qs]
            sv[b, :, j] = vn[b, :, j - qs]
    scale = 1.0 / math.sqrt(d)
    tq, tkn, tvn, trk, trv = (to_dev(x) for x in (q, kn, vn, rk, rv))
    out, lse = swa.swa_attn_chunk_ring(tq, tkn, tvn, trk, trv,
                                       torch.tensor(starts, dtype=torch.int64, device="cuda"),
                                       scale, return_lse=True, k_sink=to_dev(sk),
                                       v_sink=to_dev(sv))
    assert swa.swa_get_device_status() == 0
    ref, ref_lse = oracle.swa_chunk_sink(q, kn, vn, rk, rv, sk, sv, starts, W, scale,
                                         with_lse=True)
    assert_close_bf16out(to_f64(out), ref, what="chunk with sinks")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3


def test_chunk_sink_workload_sampled_rows(swa):
    """The benchmarked chunk-ring workload with 4 sinks, sampled rows."""
    from swa_inputs.workloads import sink_inputs
    from tests._util import assert_close_bf16out

    w = WORKLOADS["chunk_ring_sink"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    sk, sv = sink_inputs(w)
    out = swa.swa_attn_chunk_ring(to_dev(q), to_dev(kn), to_dev(vn), to_dev(rk), to_dev(rv),
                                  torch.tensor(qs, dtype=torch.int64, device="cuda"), w.scale,
                                  k_sink=to_dev(sk), v_sink=to_dev(sv))
    assert swa.swa_get_device_status() == 0
    edges = [0, 1, 127, 128, 255, 256, 383, 384, 510, 511]
    rows = sample_rows(w.B, w.H, w.Tq, 200, seed=13, extra=edges)
    ref = oracle.swa_chunk_sink(q, kn, vn, rk, rv, sk, sv, qs, w.W, w.scale, rows=rows)
    got = to_f64(out)[rows[:, 0], rows[:, 1], rows[:, 2]]
    assert_close_bf16out(got, ref, what="chunk_ring_sink workload")


# ---------------------------------------------------------------------------------------------
# swa_attn_chunk_ring_split: the same chunk calls with a workspace, where the units of the
# last round are cut into key-range parts across the SMs and merged.  Small batches have
# few units, so here nearly every unit is split; the results must match the oracle as
# the unsplit calls do, with padding rows and the ring update unchanged in meaning.

def _run_split(swa, q, kn, vn, rk, rv, qs, scale, lens=None, sk=None, sv=None, update=False,
               fill=7.0):
    tq, tkn, tvn, trk, trv = (to_dev(x) for x in (q, kn, vn, rk, rv))
    tqs = torch.tensor(qs, dtype=torch.int64, device="cuda")
    tl = None if lens is None else torch.tensor(lens, dtype=torch.int64, device="cuda")
    out = torch.full_like(tq, fill)
    lse = torch.full(tq.shape[:3], fill, dtype=torch.float32, device="cuda")
    swa.swa_attn_chunk_ring_split(tq, tkn, tvn, trk, trv, tqs, scale, chunk_len=tl,
                                  k_sink=None if sk is None else to_dev(sk),
                                  v_sink=None if sv is None else to_dev(sv), update_ring=update,
                                  out=out, lse=lse, return_lse=True)
    assert swa.swa_get_device_status() == 0
    return out, lse, trk, trv


@pytest.mark.parametrize("B,H,Hkv,Tq,d,W,starts,lens", [
    (4, 4, 2, 300, 128, 256, [512, 40, 0, 700], [300, 1, 129, 0]),
    (3, 6, 2, 256, 64, 128, [1000, 3, 129], [200, 256, 65]),
    (3, 8, 2, 384, 128, 512, [12288 + 37, 0, 511], [127, 128, 383]),
    (2, 8, 2, 512, 128, 4096, [12288, 9000], [512, 512]),       # every chunk full
])
def test_split_ragged_chunks_per_sequence(swa, B, H, Hkv, Tq, d, W, starts, lens):
    seed = 1900 + Tq + W
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    scale = 1.0 / math.sqrt(d)
    out, lse, trk, trv = _run_split(swa, q, kn, vn, rk, rv, starts, scale, lens=lens,
                                    update=True)
    got, got_lse = to_f64(out), to_f64(lse)
    erk, erv = rk.copy(), rv.copy()
    for b, (qs, n) in enumerate(zip(starts, lens)):
        assert np.all(got[b, :, n:] == 7.0)
        assert np.all(got_lse[b, :, n:] == 7.0)
        if n == 0:
            continue
        sl = (slice(b, b + 1), slice(None), slice(0, n))
        ref, ref_lse = oracle.swa_chunk(q[sl], kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [qs], W,
                                        scale, with_lse=True)
        assert_close(got[b:b + 1, :, :n], ref, what=f"split chunk b={b} len={n}")
        assert np.max(np.abs(got_lse[b:b + 1, :, :n] - ref_lse)) < 1e-3
        k1, v1 = oracle.ring_update(kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [qs], W)
        erk[b:b + 1], erv[b:b + 1] = k1, v1
    assert np.array_equal(to_host_bits(trk), erk)
    assert np.array_equal(to_host_bits(trv), erv)


@pytest.mark.parametrize("B,H,Hkv,Tq,d,W,S,starts", [
    (2, 8, 2, 200, 128, 256, 4, [5000 + 77, 300]),
    (3, 6, 2, 130, 64, 100, 16, [1000, 77, 3]),
])
def test_split_chunk_with_sinks(swa, B, H, Hkv, Tq, d, W, S, starts):
    from tests._util import assert_close_bf16out

    seed = 2100 + Tq + W + S
    q = si.normal_bf16(seed, si.STREAM["q"], (B, H, Tq, d))
    kn = si.normal_bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d))
    vn = si.normal_bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d))
    rk, rv = _ring_from_history(seed, B, Hkv, W, d, starts)
    sk = si.normal_bf16(seed, si.STREAM["k_sink"], (B, Hkv, S, d))
    sv = si.normal_bf16(seed, si.STREAM["v_sink"], (B, Hkv, S, d))
    for b, qs in enumerate(starts):
        for j in range(qs, min(S, qs + Tq)):
            sk[b, :, j] = kn[b, :, j - qs]
            sv[b, :, j] = vn[b, :, j - qs]
    scale = 1.0 / math.sqrt(d)
    out, lse, _, _ = _run_split(swa, q, kn, vn, rk, rv, starts, scale, sk=sk, sv=sv)
    ref, ref_lse = oracle.swa_chunk_sink(q, kn, vn, rk, rv, sk, sv, starts, W, scale,
                                         with_lse=True)
    assert_close_bf16out(to_f64(out), ref, what="split chunk with sinks")
    assert np.max(np.abs(to_f64(lse) - ref_lse)) < 1e-3


def test_split_ragged_workload_every_valid_row(swa):
    """The benchmarked ragged batch (1..512 valid rows per sequence) through the split call:
    every valid output row against the oracle, padding untouched."""
    from swa_inputs.workloads import seq_lens

    w = WORKLOADS["chunk_ring_ragged"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    lens = [int(n) for n in seq_lens(w)]
    out, _, _, _ = _run_split(swa, q, kn, vn, rk, rv, list(qs), w.scale, lens=lens)
    got = to_f64(out)
    for b, n in enumerate(lens):
        sl = (slice(b, b + 1), slice(None), slice(0, n))
        ref = oracle.swa_chunk(q[sl], kn[sl], vn[sl], rk[b:b + 1], rv[b:b + 1], [int(qs[b])],
                               w.W, w.scale)
        assert_close(got[b:b + 1, :, :n], ref, what=f"split ragged workload b={b}")
        assert np.all(got[b, :, n:] == 7.0)


def test_split_workload_matches_unsplit_call(swa):
    """The chunk-ring workload through both calls: within the tolerance of each other
    (the split changes only the summation order of the units it cuts)."""
    w = WORKLOADS["chunk_ring"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    a = to_f64(_run(swa, q, kn, vn, rk, rv, list(qs), w.scale)[0])
    b = to_f64(_run_split(swa, q, kn, vn, rk, rv, list(qs), w.scale)[0])
    assert_close(b, a, what="split vs unsplit")


def test_split_rejects_small_workspace(swa):
    from sliding_window_sparse_b200._native import SwaError

    B, H, Hkv, Tq, d, W = 1, 2, 2, 16, 64, 32
    z = torch.zeros((B, H, Tq, d), dtype=torch.bfloat16, device="cuda")
    zk = torch.zeros((B, Hkv, Tq, d), dtype=torch.bfloat16, device="cuda")
    rk = torch.zeros((B, Hkv, W, d), dtype=torch.bfloat16, device="cuda")
    qs = torch.tensor([40], dtype=torch.int64, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(SwaError):
        swa.swa_attn_chunk_ring_split(z, zk, zk, rk, rk.clone(), qs, 0.1, workspace=ws)
