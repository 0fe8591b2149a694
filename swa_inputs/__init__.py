"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module holds no attention arithmetic. It only turns (seed, stream id,
count) into reproducible numbers:

* ``splitmix64`` is the counter-based SplitMix64 mixer of Steele, Lea and
  Flood ("Fast splittable pseudorandom number generators", OOPSLA 2014):
  word ``i`` of a stream is the mixer applied to ``base + (i + 1) * gamma``.
* ``normal_bf16`` draws N(0, 1) values with the Box-Muller transform from
  pairs of 53-bit uniforms, rounds them to float32 and then to bfloat16 with
  round-to-nearest-even, and returns the raw bfloat16 bit patterns as
  ``uint16``.  Both the oracle and the CUDA path consume exactly those bits,
  so the rounding recipe is a definition of the input, not a precision claim.
* ``uniform_int`` draws integers in ``[lo, hi]`` (used for decode context
  lengths).

Every tensor of a workload has its own stream id, so the values of one tensor
do not depend on the sizes of the others.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "splitmix64",
    "stream_base",
    "uniform01",
    "normal_f64",
    "normal_bf16",
    "bf16_bits_to_f32",
    "f32_to_bf16_bits",
    "uniform_int",
    "STREAM",
]

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids of the tensors of a workload (one independent stream each).
STREAM = {
    "q": 1,
    "k": 2,
    "v": 3,
    "k_ring": 4,
    "v_ring": 5,
    "k_new": 6,
    "v_new": 7,
    "ctx_len": 8,
    "extra": 9,
    "seq_len": 10,
    "k_sink": 11,
    "v_sink": 12,
}


def splitmix64(x: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser applied element-wise to uint64 counters."""
    z = np.asarray(x, dtype=np.uint64).copy()
    with np.errstate(over="ignore"):
        z ^= z >> np.uint64(30)
        z *= _M1
        z ^= z >> np.uint64(27)
        z *= _M2
        z ^= z >> np.uint64(31)
    return z


def stream_base(seed: int, stream: int) -> np.uint64:
    """Start state of stream ``stream`` under ``seed`` (itself SplitMix64-mixed)."""
    key = np.array([(int(seed) & 0xFFFFFFFF) << 32 | (int(stream) & 0xFFFFFFFF)], dtype=np.uint64)
    return splitmix64(key)[0]


def _words(seed: int, stream: int, count: int, offset: int = 0) -> np.ndarray:
    base = stream_base(seed, stream)
    idx = np.arange(offset + 1, offset + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        ctr = base + idx * _GAMMA
    return splitmix64(ctr)


def uniform01(seed: int, stream: int, count: int, offset: int = 0) -> np.ndarray:
    """Uniform doubles in (0, 1]: ((w >> 11) + 1) * 2**-53."""
    w = _words(seed, stream, count, offset)
    return ((w >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)


def normal_f64(seed: int, stream: int, count: int) -> np.ndarray:
    """``count`` standard normal doubles (Box-Muller on consecutive uniform pairs)."""
    pairs = (count + 1) // 2
    u = uniform01(seed, stream, 2 * pairs)
    u1 = u[0::2]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * np.pi * u2
    out = np.empty(2 * pairs, dtype=np.float64)
    out[0::2] = r * np.cos(t)
    out[1::2] = r * np.sin(t)
    return out[:count]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = u + np.uint32(0x7FFF) + lsb
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(seed: int, stream: int, shape, scale: float = 1.0) -> np.ndarray:
    """bfloat16 bit patterns (uint16, C order) of ``scale * N(0,1)`` draws."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    vals = normal_f64(seed, stream, n) * float(scale)
    return f32_to_bf16_bits(vals.astype(np.float32)).reshape(shape)


def uniform_int(seed: int, stream: int, count: int, lo: int, hi: int) -> np.ndarray:
    """``count`` integers uniform in [lo, hi] (inclusive), as int64 (modulo reduction)."""
    span = np.uint64(int(hi) - int(lo) + 1)
    w = _words(seed, stream, count)
    return (w % span).astype(np.int64) + np.int64(lo)
