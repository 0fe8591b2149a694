"""Benchmark of the sliding-window attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]

One step is one tile-skipping prefill forward (block metadata evaluated inside
the kernel, S = QK^T and O += PV on the tensor cores, online softmax, masked
boundary tiles) over the Mistral-7B-shaped workload: B=1, H=32 query heads,
Hkv=8, N=8192, d=128, W=4096, bf16 i.i.d. N(0,1) inputs.  `value` is useful
TFLOP/s = 4 * d * valid_pairs * H * B / time, summed over ranks (each rank runs
its own independent batch: weak scaling, no data-path collective).

The same run also times the chunked-prefill-on-ring and decode paths (and the
narrow-window prefill), then the packed variable-length prefill, prefill and
decode with attention sinks, ragged chunks and the backward pass, each on its
own workload, under "paths".  It prints one JSON line
on rank 0, and adds the roofline fraction of the timed kernel, a CPU baseline
(the fp64 oracle on a bounded sample of rows, timed on the host cores), an
end-to-end figure through the public API with host buffers, and SM clocks
sampled during the timed region.

`--impl reference` times the oracle alone (on rank 0; other ranks exit).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from swa_inputs.workloads import WORKLOADS  # noqa: E402

FLUSH_BYTES = 256 << 20  # > 126 MB L2: written between timed steps
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HEADLINE = "mistral_prefill"
# workloads whose "paths" entry also times the oracle on a sample (rank 0, one GPU)
CPU_BASELINE_PATHS = ("mistral_prefill", "narrow_window", "chunk_ring", "decode_ring")
METRIC = "SWA prefill useful TFLOP/s and decode KV GB/s at 1 B200, % of roofline"


# ----------------------------------------------------------------------------- metric arithmetic

def valid_pairs_row(pos: int, W: int) -> int:
    """Allowed keys of a query at logical position pos (keys max(0, pos-W+1)..pos)."""
    return min(W, pos + 1)


def sequence_pairs(N: int, W: int, S: int = 0) -> int:
    """Visible (query, key) pairs of one sequence of N positions: N*W - W*(W-1)/2
    window pairs (N >= W), plus min(S, i - W + 1) sinks before the window of
    each query i >= W."""
    base = N * W - W * (W - 1) // 2 if N >= W else N * (N + 1) // 2
    m = max(0, N - W)
    return base + (m * (m + 1) // 2 if m <= S else S * (S + 1) // 2 + (m - S) * S)


def chunk_rows(w):
    """Valid chunk rows per sequence."""
    from swa_inputs.workloads import seq_lens

    return [int(n) for n in seq_lens(w)] if w.len_hi else [w.Tq] * w.B


def useful_flops(w) -> int:
    """4 * d * (visible pairs) * H, summed over the batch."""
    if w.kind == "prefill":
        return 4 * w.d * w.H * w.B * sequence_pairs(w.N, w.W, w.n_sink)
    if w.kind == "backward":
        # five matrix products per visible pair (S, dP, dV, dK, dQ) against the forward's two
        return 10 * w.d * w.H * w.B * sequence_pairs(w.N, w.W)
    if w.kind == "varlen":
        from swa_inputs.workloads import seq_lens

        return 4 * w.d * w.H * sum(sequence_pairs(int(n), w.W, w.n_sink) for n in seq_lens(w))
    if w.kind == "varlen_backward":
        from swa_inputs.workloads import seq_lens

        return 10 * w.d * w.H * sum(sequence_pairs(int(n), w.W, w.n_sink) for n in seq_lens(w))
    if w.kind == "chunk":
        pairs = sum(valid_pairs_row(w.q_start + t, w.W) +
                    min(w.n_sink, max(0, w.q_start + t - w.W + 1))
                    for n in chunk_rows(w) for t in range(n))
        return 4 * w.d * w.H * pairs
    raise ValueError(w.kind)


def decode_positions(w):
    from swa_inputs import STREAM, uniform_int

    return uniform_int(w.seed, STREAM["ctx_len"], w.B, w.ctx_lo, w.ctx_hi) - 1


def decode_kv_bytes(w) -> int:
    """K and V of every (b, kv head) read once: 2 tensors * B * Hkv * W * d * 2 bytes,
    plus the sink rows that lie before each window."""
    sinks = 0
    if w.n_sink:
        sinks = sum(min(w.n_sink, max(0, int(p) - w.W + 1)) for p in decode_positions(w))
    return 2 * w.Hkv * w.d * 2 * (w.B * w.W + sinks)


def algorithmic_bytes(w) -> int:
    """Compulsory HBM bytes of one call: inputs read once, outputs written once."""
    e = 2
    if w.kind == "prefill":
        return e * w.d * w.B * (2 * w.H * w.N + 2 * w.Hkv * w.N)
    if w.kind == "backward":
        # read q, k, v, out, dout (and lse); write dq, dk, dv
        return e * w.d * w.B * (4 * w.H * w.N + 4 * w.Hkv * w.N) + 4 * w.B * w.H * w.N
    if w.kind == "varlen":
        from swa_inputs.workloads import cu_seqlens

        total = int(cu_seqlens(w)[-1])
        return e * w.d * (2 * w.H * total + 2 * w.Hkv * total)
    if w.kind == "varlen_backward":
        from swa_inputs.workloads import cu_seqlens

        total = int(cu_seqlens(w)[-1])
        return e * w.d * (4 * w.H * total + 4 * w.Hkv * total) + 4 * w.H * total
    if w.kind == "chunk":
        rows = sum(chunk_rows(w))
        return e * w.d * (2 * w.H * rows + 2 * w.Hkv * (rows + w.B * w.W))
    return decode_kv_bytes(w) + e * w.d * w.B * w.H * 2


# ----------------------------------------------------------------------------- ranks

def rank_seed_offset(rank: int) -> int:
    """Each rank draws its own batch (weak scaling): the workload seed plus the rank."""
    return rank


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The slowest rank's figure (the job's time); all ranks get it."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(work_per_rank: float, world: int, ms_per_step: float, unit_div: float) -> float:
    """Whole-job throughput: every rank's work divided by the slowest rank's time."""
    return work_per_rank * world / (ms_per_step * 1e-3) / unit_div


# ----------------------------------------------------------------------------- helpers

def describe(w) -> str:
    sink = f" sinks{w.n_sink}" if w.n_sink else ""
    if w.kind in ("prefill", "backward"):
        return f"{w.name}: B{w.B} H{w.H} Hkv{w.Hkv} N{w.N} d{w.d} W{w.W}{sink}"
    if w.kind in ("varlen", "varlen_backward"):
        return (f"{w.name}: {w.n_seq} packed sequences, lengths U[{w.len_lo},{w.len_hi}], "
                f"H{w.H} Hkv{w.Hkv} d{w.d} W{w.W}{sink}")
    if w.kind == "chunk":
        rows = f" valid rows U[{w.len_lo},{w.len_hi}]" if w.len_hi else ""
        return (f"{w.name}: B{w.B} H{w.H} Hkv{w.Hkv} Tq{w.Tq} d{w.d} W{w.W} "
                f"q_start{w.q_start}{rows}{sink}")
    return (f"{w.name}: B{w.B} H{w.H} Hkv{w.Hkv} d{w.d} W{w.W} "
            f"ctx U[{w.ctx_lo},{w.ctx_hi}]{sink}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "fwd2_kernel": ("swa_fwd2.cuh", "swa_tile.cuh", "swa_epilogue.cuh", "sm100.cuh"),
    "decode_split_kernel": ("swa_decode.cuh", "sm100.cuh"),
    "bwd_kernels": ("swa_bwd.cuh", "swa_epilogue.cuh", "sm100.cuh"),
}


def kernel_source_hash(kernel: str) -> str:
    """sha256 (16 hex) of the source files a kernel is compiled from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sliding_window_sparse_b200", "csrc")
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    s = re.search(r"kernel_source_hash:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != kernel_source_hash(kernel):
        return None
    return int(m.group(1))


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons, with host timestamps."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", gpu_id, "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm = float(parts[1])
                smax = float(parts[2])
            except ValueError:
                continue
            reasons = [n for n, v in zip(self.NAMES, parts[5:9]) if v.lower().startswith("active")]
            self.samples.append((time.time(), sm, smax, reasons))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        src = "timed region"
        if len(inside) < 2:
            inside = [s for s in self.samples if s[0] <= t1]
            src = "warm-up and timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = sorted({r for s in inside for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in inside),
                "sm_max_mhz": max(s[2] for s in inside), "reasons": reasons,
                "samples": len(inside), "window": src}


# ----------------------------------------------------------------------------- inputs

def make_inputs(w, device, seed_offset=0):
    import torch

    from swa_inputs import STREAM
    from swa_inputs.torch_gen import normal_bf16_cuda

    s = w.seed + seed_offset
    g = lambda name, shape: normal_bf16_cuda(s, STREAM[name], shape, device)  # noqa: E731
    if w.kind == "prefill":
        return {"q": g("q", (w.B, w.H, w.N, w.d)), "k": g("k", (w.B, w.Hkv, w.N, w.d)),
                "v": g("v", (w.B, w.Hkv, w.N, w.d))}
    if w.kind == "backward":
        import sliding_window_sparse_b200 as swa

        x = {"q": g("q", (w.B, w.H, w.N, w.d)), "k": g("k", (w.B, w.Hkv, w.N, w.d)),
             "v": g("v", (w.B, w.Hkv, w.N, w.d)), "dout": g("extra", (w.B, w.H, w.N, w.d))}
        # the forward's output and LSE are inputs of the backward (made once, untimed)
        x["out"], x["lse"] = swa.swa_attn_fwd(x["q"], x["k"], x["v"], w.W, w.scale,
                                              return_lse=True)
        return x
    if w.kind in ("varlen", "varlen_backward"):
        from swa_inputs.workloads import cu_seqlens, seq_lens

        cu = cu_seqlens(w)
        total = int(cu[-1])
        x = {"q": g("q", (total, w.H, w.d)), "k": g("k", (total, w.Hkv, w.d)),
             "v": g("v", (total, w.Hkv, w.d)),
             "cu_seqlens": torch.tensor(cu, dtype=torch.int64, device=device)}
        if w.kind == "varlen_backward":
            import sliding_window_sparse_b200 as swa

            x["dout"] = g("extra", (total, w.H, w.d))
            # the forward's output and LSE are inputs of the backward (made once, untimed)
            x["out"], x["lse"] = swa.swa_attn_varlen(x["q"], x["k"], x["v"], x["cu_seqlens"],
                                                     int(max(seq_lens(w))), w.W, w.scale,
                                                     n_sink=w.n_sink, return_lse=True)
        return x
    if w.kind == "chunk":
        x = {"q": g("q", (w.B, w.H, w.Tq, w.d)),
             "k_new": g("k_new", (w.B, w.Hkv, w.Tq, w.d)),
             "v_new": g("v_new", (w.B, w.Hkv, w.Tq, w.d)),
             "k_ring": g("k_ring", (w.B, w.Hkv, w.W, w.d)),
             "v_ring": g("v_ring", (w.B, w.Hkv, w.W, w.d)),
             "q_start": torch.full((w.B,), w.q_start, dtype=torch.int64, device=device)}
        if w.len_hi:
            x["chunk_len"] = torch.tensor(chunk_rows(w), dtype=torch.int64, device=device)
        if w.n_sink:
            x["k_sink"] = g("k_sink", (w.B, w.Hkv, w.n_sink, w.d))
            x["v_sink"] = g("v_sink", (w.B, w.Hkv, w.n_sink, w.d))
        return x
    from swa_inputs import uniform_int

    ctx = uniform_int(s, STREAM["ctx_len"], w.B, w.ctx_lo, w.ctx_hi)
    x = {"q": g("q", (w.B, w.H, w.d)), "k_ring": g("k_ring", (w.B, w.Hkv, w.W, w.d)),
         "v_ring": g("v_ring", (w.B, w.Hkv, w.W, w.d)),
         "pos": torch.tensor(ctx - 1, dtype=torch.int64, device=device)}
    if w.n_sink:
        x["k_sink"] = g("k_sink", (w.B, w.Hkv, w.n_sink, w.d))
        x["v_sink"] = g("v_sink", (w.B, w.Hkv, w.n_sink, w.d))
    return x


def make_call(w, x, swa):
    """The public-API call of one step on device-resident inputs."""
    import torch

    if w.kind == "prefill":
        out = torch.empty_like(x["q"])
        return (lambda: swa.swa_attn_fwd(x["q"], x["k"], x["v"], w.W, w.scale, out=out,
                                         n_sink=w.n_sink), out, 1)
    if w.kind == "backward":
        dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
        ws = torch.empty(int(swa.lib().swa_attn_bwd_workspace_bytes(w.B, w.H, w.N)),
                         dtype=torch.uint8, device=x["q"].device)
        return (lambda: swa.swa_attn_bwd(x["q"], x["k"], x["v"], x["out"], x["dout"], x["lse"],
                                         w.W, w.scale, dq=dq, dk=dk, dv=dv, workspace=ws), dq, 2)
    if w.kind == "varlen_backward":
        from swa_inputs.workloads import seq_lens

        dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
        total = x["q"].shape[0]
        ws = torch.empty(int(swa.lib().swa_attn_varlen_bwd_workspace_bytes(w.H, total)),
                         dtype=torch.uint8, device=x["q"].device)
        max_len = int(max(seq_lens(w)))
        return (lambda: swa.swa_attn_varlen_bwd(x["q"], x["k"], x["v"], x["cu_seqlens"], max_len,
                                                x["out"], x["dout"], x["lse"], w.W, w.scale,
                                                n_sink=w.n_sink, dq=dq, dk=dk, dv=dv,
                                                workspace=ws), dq, 2)
    if w.kind == "varlen":
        from swa_inputs.workloads import seq_lens

        out = torch.empty_like(x["q"])
        max_len = int(max(seq_lens(w)))
        return (lambda: swa.swa_attn_varlen(x["q"], x["k"], x["v"], x["cu_seqlens"], max_len,
                                            w.W, w.scale, n_sink=w.n_sink, out=out), out, 1)
    if w.kind == "chunk":
        out = torch.empty_like(x["q"])
        if "chunk_len" in x:
            # ragged chunks leave the last round of units part empty: the split call
            # (schedule, attention, merge) cuts those units by key range across the SMs
            ws = torch.empty(swa.swa_chunk_split_workspace_bytes(w.B, w.H, w.Hkv, w.Tq, w.d, w.W),
                             dtype=torch.uint8, device=x["q"].device)
            return (lambda: swa.swa_attn_chunk_ring_split(
                x["q"], x["k_new"], x["v_new"], x["k_ring"], x["v_ring"], x["q_start"], w.scale,
                chunk_len=x["chunk_len"], out=out, workspace=ws), out, 3)
        return (lambda: swa.swa_attn_chunk_ring(x["q"], x["k_new"], x["v_new"], x["k_ring"],
                                                x["v_ring"], x["q_start"], w.scale, out=out,
                                                k_sink=x.get("k_sink"), v_sink=x.get("v_sink")),
                out, 1)
    out = torch.empty_like(x["q"])
    ws = torch.empty(swa.swa_decode_workspace_bytes(w.B, w.H, w.Hkv, w.d, w.W), dtype=torch.uint8,
                     device=x["q"].device)
    return (lambda: swa.swa_attn_decode_ring(x["q"], x["k_ring"], x["v_ring"], x["pos"], w.scale,
                                             workspace=ws, out=out, k_sink=x.get("k_sink"),
                                             v_sink=x.get("v_sink")), out, 2)


def time_steps(call, steps, warmup, flush, barrier):
    """Per-step device time (ms) with CUDA events on the launching stream; L2 flushed
    between steps outside the timed windows."""
    import torch

    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize()
    barrier()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    t0 = time.time()
    for i in range(steps):
        flush.zero_()
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    barrier()
    return [s.elapsed_time(e) for s, e in zip(starts, ends)], t0, t1


def time_e2e(w, x, swa, steps, warmup):
    """Same metric through the public API with pinned host inputs: H2D copies, the call
    and the D2H copy of the result inside the timed window."""
    import torch

    dev = x["q"].device
    names = [n for n in x if x[n].dtype != torch.int64]  # positions and offsets stay put
    host = {n: x[n].cpu().pin_memory() for n in names}
    xs = dict(x)
    call, out, _ = make_call(w, xs, swa)
    out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    stream = torch.cuda.current_stream()
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = out.numel() * out.element_size()

    def step():
        for n in names:
            xs[n].copy_(host[n], non_blocking=True)
        call()
        out_host.copy_(out, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    del dev
    return e0.elapsed_time(e1) / steps, h2d, d2h


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(w, host_inputs, n_rows, seed=12345):
    """Time the oracle on a sample of workload w: n_rows random query rows (prefill,
    chunk) or n_rows sequences (decode).  Returns (seconds, work) with work in the
    workload's unit: useful FLOPs, or K/V bytes read for decode."""
    import oracle

    rng = np.random.default_rng(seed)
    if w.kind == "prefill":
        q, k, v = host_inputs
        rows = np.stack([rng.integers(w.B, size=n_rows), rng.integers(w.H, size=n_rows),
                         rng.integers(w.N, size=n_rows)], axis=1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.swa_forward(q, k, v, w.W, w.scale, rows=rows)
        dt = time.perf_counter() - t0
        pairs = sum(valid_pairs_row(int(i), w.W) for i in rows[:, 2])
        return dt, 4 * w.d * pairs
    if w.kind == "chunk" and not w.len_hi and not w.n_sink:
        q, kn, vn, rk, rv, qs = host_inputs
        rows = np.stack([rng.integers(w.B, size=n_rows), rng.integers(w.H, size=n_rows),
                         rng.integers(w.Tq, size=n_rows)], axis=1).astype(np.int64)
        t0 = time.perf_counter()
        oracle.swa_chunk(q, kn, vn, rk, rv, qs, w.W, w.scale, rows=rows)
        dt = time.perf_counter() - t0
        pairs = sum(valid_pairs_row(int(qs[b]) + int(t), w.W) for b, _, t in rows)
        return dt, 4 * w.d * pairs
    if w.kind == "decode" and not w.n_sink:
        q, rk, rv, pos = host_inputs
        sel = np.sort(rng.choice(w.B, size=min(n_rows, w.B), replace=False))
        args = [np.ascontiguousarray(a[sel]) for a in (q, rk, rv)]
        t0 = time.perf_counter()
        oracle.swa_decode(*args, pos[sel], w.W, w.scale)
        dt = time.perf_counter() - t0
        return dt, 2 * w.Hkv * w.d * 2 * w.W * len(sel)
    raise ValueError(w.kind)


def sample_units(w) -> int:
    """Most sample units oracle_sample can draw: query rows, or sequences for decode."""
    if w.kind == "decode":
        return w.B
    if w.kind == "chunk":
        return w.B * w.H * w.Tq
    return w.B * w.H * w.N


def calibrated_oracle(w, host_inputs, seconds):
    """Grow the sample until one oracle pass takes about `seconds`."""
    n = 16 if w.kind != "decode" else 1
    dt, fl = oracle_sample(w, host_inputs, n)
    while dt < seconds / 4 and n < sample_units(w):
        n = min(sample_units(w), int(n * max(2.0, (seconds / max(dt, 1e-3)) * 0.9)))
        dt, fl = oracle_sample(w, host_inputs, n)
    return dt, fl, n


def host_inputs_of(w, x):
    """Host (numpy) copies of a workload's device inputs in the oracle's argument order."""
    import torch

    def bits(t):
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)

    if w.kind == "prefill":
        return tuple(bits(x[n]) for n in ("q", "k", "v"))
    if w.kind == "chunk":
        return tuple(bits(x[n]) for n in ("q", "k_new", "v_new", "k_ring", "v_ring")) + \
            (x["q_start"].cpu().numpy(),)
    return tuple(bits(x[n]) for n in ("q", "k_ring", "v_ring")) + (x["pos"].cpu().numpy(),)


def cpu_baseline(w, host, seconds):
    """The oracle timed on a calibrated sample of workload w, on all host cores."""
    import oracle

    dt, work, n = calibrated_oracle(w, host, seconds)
    if w.kind == "decode":
        return {"value": work / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
                "kind": "oracle",
                "sample": f"{n} random sequences of {w.name} (whole ring each), {dt:.1f} s"}
    return {"value": work / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{n} random query rows of {w.name} (full window each), {dt:.1f} s"}


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle

    w = WORKLOADS[HEADLINE]
    from swa_inputs.workloads import prefill_inputs

    host = prefill_inputs(w)
    budget = 90.0
    per_step = max(0.2, budget / max(1, args.steps + args.warmup))
    dt, fl, n_rows = calibrated_oracle(w, host, per_step)
    for i in range(args.warmup):
        oracle_sample(w, host, n_rows, seed=100 + i)
    tot_t, tot_f = 0.0, 0
    for i in range(args.steps):
        dt, fl = oracle_sample(w, host, n_rows, seed=1000 + i)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(w),
                   "sample": f"{n_rows} random query rows per step, full window each"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(),
                         "kind": "oracle",
                         "sample": f"{n_rows} rows x {args.steps} steps of the {HEADLINE} workload"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


def run_native(args):
    import torch
    import torch.distributed as dist

    import sliding_window_sparse_b200 as swa

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def job_max(x):
        return max_over_ranks(x, world, dev)

    peaks, peak_src = load_peaks()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    props = torch.cuda.get_device_properties(dev)
    gpu_id = f"GPU-{props.uuid}" if getattr(props, "uuid", None) else str(local)
    sampler = ClockSampler(gpu_id) if rank == 0 else None

    # headline (default: the Mistral-shaped prefill), each rank its own batch
    headline = args.workload
    w = WORKLOADS[headline]
    x = make_inputs(w, dev, seed_offset=rank_seed_offset(rank))
    call, out, launches_per_step = make_call(w, x, swa)
    times, t0, t1 = time_steps(call, args.steps, args.warmup, flush, barrier)
    if swa.swa_get_device_status() != 0:
        raise SystemExit("device status error during the timed region")
    total_ms = job_max(sum(times))
    mean_ms = total_ms / args.steps
    if w.kind == "decode":
        work, unit, scale_div, bound, peak = decode_kv_bytes(w), "GB/s", 1e9, "hbm", "hbm_gbs"
    else:
        work, unit, scale_div, bound, peak = useful_flops(w), "TFLOP/s", 1e12, "tensor", "bf16_tflops"
    value = job_rate(work, world, mean_ms, scale_div)
    kernel_rate = work / (statistics.mean(times) * 1e-3) / scale_div
    clocks = sampler.summary(t0, t1) if sampler else None

    # end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, 20))
    e2e_ms, h2d, d2h = time_e2e(w, x, swa, e2e_steps, 2)
    e2e_ms = job_max(e2e_ms)
    e2e_value = job_rate(work, world, e2e_ms, scale_div)

    # the other paths of the hot path, on their own workloads
    paths = {}
    if not args.headline_only:
        for name in ("mistral_prefill", "narrow_window", "chunk_ring", "decode_ring",
                     "varlen_prefill", "mistral_prefill_sink", "chunk_ring_ragged",
                     "decode_ring_sink", "chunk_ring_sink", "mistral_backward",
                     "varlen_backward"):
            if name == headline:
                continue
            pw = WORKLOADS[name]
            px = make_inputs(pw, dev, seed_offset=rank_seed_offset(rank))
            pcall, _, nl = make_call(pw, px, swa)
            psteps = max(10, min(args.steps, 200))
            ptimes, _, _ = time_steps(pcall, psteps, max(3, args.warmup), flush, barrier)
            pms = job_max(sum(ptimes)) / psteps
            entry = {"workload": name, "ms_per_call": pms, "launches_per_call": nl}
            if pw.kind == "decode":
                gbs = decode_kv_bytes(pw) / (pms * 1e-3) / 1e9
                entry.update({"value": gbs * world, "unit": "GB/s",
                              "roofline": {"bound": "hbm", "achieved": gbs,
                                           "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                           "frac": gbs / peaks["hbm_gbs"],
                                           "traffic": profiled_traffic("decode_split_kernel",
                                                                       name),
                                           "note": "KV bytes over split+combine time"}})
            else:
                tf = useful_flops(pw) / (pms * 1e-3) / 1e12
                entry.update({"value": tf * world, "unit": "TFLOP/s",
                              "roofline": {"bound": "tensor", "achieved": tf,
                                           "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                           "frac": tf / peaks["bf16_tflops"],
                                           "traffic": profiled_traffic(
                                               "bwd_kernels" if "backward" in pw.kind
                                               else "fwd2_kernel", name)}})
            if (rank == 0 and world == 1 and not args.no_cpu_baseline
                    and name in CPU_BASELINE_PATHS):
                entry["cpu_baseline"] = cpu_baseline(pw, host_inputs_of(pw, px),
                                                     args.cpu_seconds / 3)
            paths[name] = entry
            del px, pcall
            torch.cuda.empty_cache()

    if sampler:
        sampler.stop()

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline and headline in CPU_BASELINE_PATHS:
            cpu = cpu_baseline(w, host_inputs_of(w, x), args.cpu_seconds)
        kname = "decode_split_kernel" if w.kind == "decode" else "fwd2_kernel"
        roof = {"bound": bound, "achieved": kernel_rate, "peak": peaks[peak], "unit": unit,
                "frac": kernel_rate / peaks[peak],
                "traffic": profiled_traffic(kname, headline),
                "peak_source": f"{peak_src} " + ("bf16 burst" if bound == "tensor" else "copy"),
                "algorithmic_bytes": algorithmic_bytes(w)}
        if bound == "tensor":
            roof["frac_of_sustained"] = kernel_rate / peaks["bf16_tflops_sustained"]
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": describe(w), "batch": "one batch per rank",
                       "work_per_step": work, "l2": "flushed by a 256 MiB write "
                       "between timed steps"},
            "roofline": roof, "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * launches_per_step,
            "clocks": clocks, "paths": paths,
        }
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--headline-only", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE,
                    help="headline workload (default: the Mistral-shaped prefill)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_native(args)


if __name__ == "__main__":
    sys.exit(main())
