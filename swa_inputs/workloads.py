"""The synthetic workloads: shapes, seeds and value recipes (no attention arithmetic).

Every tensor is bf16 i.i.d. N(0, 1) from :func:`swa_inputs.normal_bf16` with the
workload's seed and the tensor's own stream id.  Decode context lengths, packed
sequence lengths and ragged chunk lengths are uniform integers from the same
generator.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import STREAM, normal_bf16, uniform_int


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "prefill" | "chunk" | "decode"
    B: int
    H: int
    Hkv: int
    d: int
    W: int
    N: int = 0         # prefill sequence length
    Tq: int = 0        # chunk length
    q_start: int = 0   # chunk start (same for every sequence)
    ctx_lo: int = 0    # decode context length range (inclusive)
    ctx_hi: int = 0
    n_sink: int = 0    # attention sinks: positions 0 .. n_sink-1 stay visible
    n_seq: int = 0     # varlen: sequences in the packed batch
    len_lo: int = 0    # varlen sequence / ragged chunk length range (inclusive)
    len_hi: int = 0
    seed: int = 0
    note: str = field(default="", compare=False)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# The five workloads (seed = index).
WORKLOADS = {
    "tiny": Workload("tiny", "prefill", B=1, H=4, Hkv=4, d=64, W=64, N=512, seed=0,
                     note="tiny SWA forward, parity only"),
    "mistral_prefill": Workload("mistral_prefill", "prefill", B=1, H=32, Hkv=8, d=128, W=4096,
                                N=8192, seed=1, note="Mistral-7B-shaped prefill, GQA 4"),
    "narrow_window": Workload("narrow_window", "prefill", B=2, H=32, Hkv=32, d=128, W=512,
                              N=32768, seed=2, note="long prefill, narrow window"),
    "chunk_ring": Workload("chunk_ring", "chunk", B=4, H=32, Hkv=8, d=128, W=4096, Tq=512,
                           q_start=12288, seed=3, note="chunked prefill on a ring cache"),
    "decode_ring": Workload("decode_ring", "decode", B=64, H=32, Hkv=8, d=128, W=4096,
                            ctx_lo=4096, ctx_hi=131072, seed=4, note="batched decode"),
    # the next rows: packed variable-length prefill, sinks, ragged chunks
    "varlen_prefill": Workload("varlen_prefill", "varlen", B=1, H=32, Hkv=8, d=128, W=4096,
                               n_seq=16, len_lo=256, len_hi=16384, seed=5,
                               note="16 packed sequences of 256..16384 tokens"),
    "mistral_prefill_sink": Workload("mistral_prefill_sink", "prefill", B=1, H=32, Hkv=8, d=128,
                                     W=4096, N=8192, n_sink=4, seed=6,
                                     note="Mistral-shaped prefill with 4 attention sinks"),
    "chunk_ring_ragged": Workload("chunk_ring_ragged", "chunk", B=4, H=32, Hkv=8, d=128, W=4096,
                                  Tq=512, q_start=12288, len_lo=1, len_hi=512, seed=7,
                                  note="chunks of 1..512 valid rows on a ring cache"),
    "decode_ring_sink": Workload("decode_ring_sink", "decode", B=64, H=32, Hkv=8, d=128, W=4096,
                                 ctx_lo=4096, ctx_hi=131072, n_sink=4, seed=8,
                                 note="batched decode with 4 attention sinks"),
    "chunk_ring_sink": Workload("chunk_ring_sink", "chunk", B=4, H=32, Hkv=8, d=128, W=4096,
                                Tq=512, q_start=12288, n_sink=4, seed=10,
                                note="chunked prefill on a ring cache with 4 attention sinks"),
    "varlen_backward": Workload("varlen_backward", "varlen_backward", B=1, H=32, Hkv=8, d=128,
                                W=4096, n_seq=16, len_lo=256, len_hi=16384, n_sink=4, seed=11,
                                note="gradients of 16 packed sequences with 4 sinks"),
    "mistral_backward": Workload("mistral_backward", "backward", B=1, H=32, Hkv=8, d=128, W=4096,
                                 N=8192, seed=9, note="gradients of the Mistral-shaped prefill"),
}


def seq_lens(w: Workload) -> np.ndarray:
    """Packed sequence lengths (varlen) or valid chunk rows per sequence (ragged chunk)."""
    count = w.n_seq if w.kind in ("varlen", "varlen_backward") else w.B
    return uniform_int(w.seed, STREAM["seq_len"], count, w.len_lo, w.len_hi)


def cu_seqlens(w: Workload) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(seq_lens(w))]).astype(np.int64)


def prefill_inputs(w: Workload):
    q = normal_bf16(w.seed, STREAM["q"], (w.B, w.H, w.N, w.d))
    k = normal_bf16(w.seed, STREAM["k"], (w.B, w.Hkv, w.N, w.d))
    v = normal_bf16(w.seed, STREAM["v"], (w.B, w.Hkv, w.N, w.d))
    return q, k, v


def varlen_inputs(w: Workload):
    """Token-major packed q [total, H, d], k, v [total, Hkv, d] and cu_seqlens."""
    cu = cu_seqlens(w)
    total = int(cu[-1])
    q = normal_bf16(w.seed, STREAM["q"], (total, w.H, w.d))
    k = normal_bf16(w.seed, STREAM["k"], (total, w.Hkv, w.d))
    v = normal_bf16(w.seed, STREAM["v"], (total, w.Hkv, w.d))
    return q, k, v, cu


def sink_inputs(w: Workload):
    """Sink rows [B, Hkv, n_sink, d] of a decode or chunk workload."""
    k = normal_bf16(w.seed, STREAM["k_sink"], (w.B, w.Hkv, w.n_sink, w.d))
    v = normal_bf16(w.seed, STREAM["v_sink"], (w.B, w.Hkv, w.n_sink, w.d))
    return k, v


def chunk_inputs(w: Workload):
    q = normal_bf16(w.seed, STREAM["q"], (w.B, w.H, w.Tq, w.d))
    k_ring = normal_bf16(w.seed, STREAM["k_ring"], (w.B, w.Hkv, w.W, w.d))
    v_ring = normal_bf16(w.seed, STREAM["v_ring"], (w.B, w.Hkv, w.W, w.d))
    k_new = normal_bf16(w.seed, STREAM["k_new"], (w.B, w.Hkv, w.Tq, w.d))
    v_new = normal_bf16(w.seed, STREAM["v_new"], (w.B, w.Hkv, w.Tq, w.d))
    q_start = np.full(w.B, w.q_start, dtype=np.int64)
    return q, k_new, v_new, k_ring, v_ring, q_start


def decode_inputs(w: Workload):
    q = normal_bf16(w.seed, STREAM["q"], (w.B, w.H, w.d))
    k_ring = normal_bf16(w.seed, STREAM["k_ring"], (w.B, w.Hkv, w.W, w.d))
    v_ring = normal_bf16(w.seed, STREAM["v_ring"], (w.B, w.Hkv, w.W, w.d))
    ctx = uniform_int(w.seed, STREAM["ctx_len"], w.B, w.ctx_lo, w.ctx_hi)
    pos = ctx - 1  # the query is the last token of its context
    return q, k_ring, v_ring, pos
