"""Every output element of the Mistral-shaped prefill, the narrow-window prefill
and the chunk-on-ring workload (and of their variants with 4 attention sinks)
against the fp64 oracle; and, for the Mistral-shaped backward, every gradient
element of one key/value head group at the full size.

The tolerance is the one stated for these workloads: max-abs 1e-2 and mean-abs
1e-3 over the whole tensor (bf16 inputs, fp32 accumulation, bf16 output), plus
a relative RMS bound because outputs with W in the thousands are only ~0.02 in
size.  The oracle runs on all host cores; it is fed slices of a few heads at a
time so that its fp64 results stay a few hundred MB.
"""

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from swa_inputs.workloads import WORKLOADS, chunk_inputs, prefill_inputs, sink_inputs
from tests._util import MAX_ABS, MEAN_ABS, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


class ErrorStats:
    """Running max-abs, mean-abs and relative RMS error over slices of a tensor."""

    def __init__(self):
        self.max_abs = 0.0
        self.sum_abs = 0.0
        self.sum_sq = 0.0
        self.sum_sq_ref = 0.0
        self.count = 0

    def add(self, got, ref):
        assert np.all(np.isfinite(got)), "non-finite output"
        diff = np.abs(got - ref)
        self.max_abs = max(self.max_abs, float(diff.max()))
        self.sum_abs += float(diff.sum())
        self.sum_sq += float(np.square(diff).sum())
        self.sum_sq_ref += float(np.square(ref).sum())
        self.count += diff.size

    def check(self, what):
        mean_abs = self.sum_abs / self.count
        rel_rms = (self.sum_sq / self.sum_sq_ref) ** 0.5
        assert self.max_abs <= MAX_ABS and mean_abs <= MEAN_ABS and rel_rms < 1e-2, \
            f"{what}: max-abs {self.max_abs:.3e}, mean-abs {mean_abs:.3e}, rel-RMS {rel_rms:.3e}"


def _gpu_slice_f64(out, b, h0, h1):
    return out[b, h0:h1].float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name", ["mistral_prefill", "narrow_window"])
def test_prefill_workload_every_element(swa, name):
    w = WORKLOADS[name]
    q, k, v = prefill_inputs(w)
    out = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), w.W, w.scale)
    assert swa.swa_get_device_status() == 0
    torch.cuda.synchronize()
    G = w.H // w.Hkv
    step = 8 if w.H % 8 == 0 and 8 % G == 0 else G  # query heads per oracle call
    stats = ErrorStats()
    for b in range(w.B):
        for h0 in range(0, w.H, step):
            h1 = h0 + step
            qs = np.ascontiguousarray(q[b:b + 1, h0:h1])
            ks = np.ascontiguousarray(k[b:b + 1, h0 // G:h1 // G])
            vs = np.ascontiguousarray(v[b:b + 1, h0 // G:h1 // G])
            ref = oracle.swa_forward(qs, ks, vs, w.W, w.scale)[0]
            stats.add(_gpu_slice_f64(out, b, h0, h1), ref)
    assert stats.count == w.B * w.H * w.N * w.d
    stats.check(name)


def test_chunk_ring_workload_every_element(swa):
    w = WORKLOADS["chunk_ring"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    tqs = torch.tensor(qs, dtype=torch.int64, device="cuda")
    out = swa.swa_attn_chunk_ring(to_dev(q), to_dev(kn), to_dev(vn), to_dev(rk), to_dev(rv), tqs,
                                  w.scale)
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_chunk(q, kn, vn, rk, rv, qs, w.W, w.scale)
    stats = ErrorStats()
    stats.add(out.float().cpu().numpy().astype(np.float64), ref)
    assert stats.count == w.B * w.H * w.Tq * w.d
    stats.check("chunk_ring")


def test_sink_prefill_workload_every_element(swa):
    """Mistral-shaped prefill with 4 sinks (taxonomy page section 3.2): every element."""
    w = WORKLOADS["mistral_prefill_sink"]
    q, k, v = prefill_inputs(w)
    out = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), w.W, w.scale, n_sink=w.n_sink)
    assert swa.swa_get_device_status() == 0
    torch.cuda.synchronize()
    G = w.H // w.Hkv
    tm = lambda x: np.ascontiguousarray(x[0].transpose(1, 0, 2))  # noqa: E731  [N, heads, d]
    stats = ErrorStats()
    for h0 in range(0, w.H, 2 * G):
        h1 = h0 + 2 * G
        ref = oracle.swa_varlen(tm(q[:, h0:h1]), tm(k[:, h0 // G:h1 // G]),
                                tm(v[:, h0 // G:h1 // G]), [0, w.N], w.W, w.scale,
                                n_sink=w.n_sink)
        stats.add(_gpu_slice_f64(out, 0, h0, h1), ref.transpose(1, 0, 2))
    assert stats.count == w.B * w.H * w.N * w.d
    stats.check("mistral_prefill_sink")


def test_chunk_ring_sink_workload_every_element(swa):
    """Chunk of 512 on a full ring with 4 sink rows: every element."""
    w = WORKLOADS["chunk_ring_sink"]
    q, kn, vn, rk, rv, qs = chunk_inputs(w)
    sk, sv = sink_inputs(w)
    out = swa.swa_attn_chunk_ring(to_dev(q), to_dev(kn), to_dev(vn), to_dev(rk), to_dev(rv),
                                  torch.tensor(qs, dtype=torch.int64, device="cuda"), w.scale,
                                  k_sink=to_dev(sk), v_sink=to_dev(sv))
    assert swa.swa_get_device_status() == 0
    ref = oracle.swa_chunk_sink(q, kn, vn, rk, rv, sk, sv, qs, w.W, w.scale)
    stats = ErrorStats()
    stats.add(out.float().cpu().numpy().astype(np.float64), ref)
    assert stats.count == w.B * w.H * w.Tq * w.d
    stats.check("chunk_ring_sink")


def test_mistral_backward_one_group_every_element(swa):
    """The benchmarked backward (B1 H32 Hkv8 N8192 d128 W4096) at its full size: the
    gradients of key/value head 0's group (dq of query heads 0..G-1, dk and dv of key
    head 0) depend on that group alone, so the oracle differentiates the group's slice
    and every element of those gradients is compared.  Bounds per gradient tensor as
    in the backward tests: max-abs <= 8u max|ref|, mean-abs <= 2u mean|ref|, relative
    RMS <= 1e-2 (u = 2^-8)."""
    w = WORKLOADS["mistral_backward"]
    q, k, v = prefill_inputs(w)
    g = si.normal_bf16(w.seed, si.STREAM["extra"], q.shape)
    tq, tk, tv, tg = to_dev(q), to_dev(k), to_dev(v), to_dev(g)
    out, lse = swa.swa_attn_fwd(tq, tk, tv, w.W, w.scale, return_lse=True)
    dq, dk, dv = swa.swa_attn_bwd(tq, tk, tv, out, tg, lse, w.W, w.scale)
    assert swa.swa_get_device_status() == 0
    G = w.H // w.Hkv
    rq, rk, rv = oracle.swa_backward(np.ascontiguousarray(q[:, :G]), np.ascontiguousarray(k[:, :1]),
                                     np.ascontiguousarray(v[:, :1]), np.ascontiguousarray(g[:, :G]),
                                     w.W, w.scale)
    u = 2.0 ** -8
    for name, got, ref in (("dq", dq[:, :G], rq), ("dk", dk[:, :1], rk), ("dv", dv[:, :1], rv)):
        got = got.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got)), f"{name}: non-finite"
        err = np.abs(got - ref)
        mx, mn = float(err.max()), float(err.mean())
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        assert mx <= 8 * u * float(np.abs(ref).max()), f"{name}: max-abs {mx:.3e}"
        assert mn <= 2 * u * float(np.abs(ref).mean()), f"{name}: mean-abs {mn:.3e}"
        assert rel <= 1e-2, f"{name}: relative RMS {rel:.3e}"
