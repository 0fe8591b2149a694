"""Shared helpers for the GPU parity tests (host <-> device marshalling, tolerances)."""

from __future__ import annotations

import numpy as np

# Tolerances on attention outputs against the fp64 oracle (bf16 in, fp32 accumulate,
# bf16 out): element-wise max-abs and mean-abs error.
MAX_ABS = 1e-2
MEAN_ABS = 1e-3


def to_dev(a, device="cuda"):
    """numpy uint16 bf16 bits -> torch bf16 CUDA tensor (same values)."""
    import torch

    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_host_bits(t):
    """torch bf16 tensor -> numpy uint16 bits."""
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def errors(got, ref):
    diff = np.abs(np.asarray(got, dtype=np.float64) - np.asarray(ref, dtype=np.float64))
    return float(diff.max()), float(diff.mean())


def assert_close(got, ref, max_abs=MAX_ABS, mean_abs=MEAN_ABS, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mn = errors(got, ref)
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max-abs {mx:.3e}, mean-abs {mn:.3e}"
    return mx, mn


def sample_rows(B, H, n, count, seed, extra=()):
    """Sampled (b, h, i) triples: random ones plus every tile boundary row given in `extra`."""
    rng = np.random.default_rng(seed)
    rows = set()
    for i in extra:
        if 0 <= i < n:
            rows.add((int(rng.integers(B)), int(rng.integers(H)), int(i)))
    while len(rows) < count + len(extra):
        rows.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(n))))
    return np.array(sorted(rows), dtype=np.int64)
