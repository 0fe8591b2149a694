"""The same seeded generator as :mod:`swa_inputs`, evaluated with torch on a GPU.

Used where workloads are too large to draw on the host in reasonable time (the
benchmark).  SplitMix64 runs in wrapping int64 arithmetic with logical right
shifts; Box-Muller runs in float64 with the device's log/sqrt/sin/cos, so a
value can differ from the numpy draw in its last float64 bit and, rarely, in
its rounded bf16 bits.  Tests that compare against stored or host-drawn values
use the numpy generator.
"""

from __future__ import annotations

import math

import numpy as np

from . import stream_base

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _s64(x: int) -> int:
    x &= (1 << 64) - 1
    return x - (1 << 64) if x >= 1 << 63 else x


def _srl(t, k: int):
    return (t >> k) & ((1 << (64 - k)) - 1)


def _mix(z):
    z = z ^ _srl(z, 30)
    z = z * _s64(_M1)
    z = z ^ _srl(z, 27)
    z = z * _s64(_M2)
    return z ^ _srl(z, 31)


def normal_bf16_cuda(seed: int, stream: int, shape, device="cuda", chunk: int = 1 << 25):
    """bf16 tensor of N(0, 1) draws, same recipe as swa_inputs.normal_bf16."""
    import torch

    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    base = _s64(int(stream_base(seed, stream)))
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    pairs_total = (n + 1) // 2
    for p0 in range(0, pairs_total, chunk):
        p1 = min(pairs_total, p0 + chunk)
        # counters of the uniform pair k are 2k+1 and 2k+2
        idx = torch.arange(2 * p0 + 1, 2 * p1 + 1, dtype=torch.int64, device=device)
        ctr = idx * _s64(_GAMMA) + base
        w = _mix(ctr)
        u = (_srl(w, 11).to(torch.float64) + 1.0) * (2.0 ** -53)
        u1, u2 = u[0::2], u[1::2]
        r = torch.sqrt(-2.0 * torch.log(u1))
        t = 2.0 * math.pi * u2
        vals = torch.stack([r * torch.cos(t), r * torch.sin(t)], dim=1).reshape(-1)
        lo = 2 * p0
        hi = min(n, 2 * p1)
        out[lo:hi] = vals[: hi - lo].to(torch.float32).to(torch.bfloat16)
    return out.reshape(shape)


def uniform_int_host(seed: int, stream: int, count: int, lo: int, hi: int):
    from . import uniform_int

    return uniform_int(seed, stream, count, lo, hi)
