"""Guard bands around every buffer the library writes.

Each output, workspace and in-place ring of every entry point is carved out of
a larger device buffer whose margins before and after hold a sentinel bit
pattern.  After the call the margins must be bit-identical (no store strays
outside its buffer), and the guarded output must equal, bit for bit, the same
call made on plainly allocated buffers (every element the call owns was
written).  Margins are placed at two offsets, so that the guarded buffer is
once 256-byte aligned and once only 16-byte aligned, the smallest alignment
the library accepts.  The small shapes span several tiles and end in ragged
tails, where the 128-byte row-segment stores of the epilogues skip rows.
"""

import math

import numpy as np
import pytest
import torch

import swa_inputs as si
from tests._util import to_dev

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes before and after each guarded buffer (plus the offset below)
SENTINEL = 0xA5  # every margin byte


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


class Guarded:
    """A tensor of `shape` and `dtype` inside a sentinel-filled byte buffer."""

    def __init__(self, shape, dtype, offset, fill=None):
        esize = torch.empty((), dtype=dtype).element_size()
        nbytes = int(np.prod(shape)) * esize
        self.lo = MARGIN + offset
        self.hi = self.lo + nbytes
        self.raw = torch.full((self.hi + MARGIN,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.t = self.raw[self.lo:self.hi].view(dtype).view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def margins_intact(self):
        torch.cuda.synchronize()
        return bool(torch.all(self.raw[:self.lo] == SENTINEL)) and \
            bool(torch.all(self.raw[self.hi:] == SENTINEL))


OFFSETS = [0, 16]


def _bf16(seed, stream, shape):
    return to_dev(si.normal_bf16(seed, stream, shape))


@pytest.mark.parametrize("offset", OFFSETS)
@pytest.mark.parametrize("n_sink", [0, 4])
def test_prefill_out_and_lse(swa, offset, n_sink):
    B, H, Hkv, N, d, W = 2, 4, 2, 300, 128, 100
    q, k, v = (_bf16(21, s, sh) for s, sh in ((1, (B, H, N, d)), (2, (B, Hkv, N, d)),
                                               (3, (B, Hkv, N, d))))
    out = Guarded((B, H, N, d), torch.bfloat16, offset)
    lse = Guarded((B, H, N), torch.float32, offset)
    swa.swa_attn_fwd(q, k, v, W, 0.1, out=out.t, lse=lse.t, n_sink=n_sink)
    assert swa.swa_get_device_status() == 0
    assert out.margins_intact() and lse.margins_intact()
    ref, ref_lse = swa.swa_attn_fwd(q, k, v, W, 0.1, return_lse=True, n_sink=n_sink)
    assert torch.equal(out.t, ref) and torch.equal(lse.t, ref_lse)


@pytest.mark.parametrize("offset", OFFSETS)
def test_prefill_d64(swa, offset):
    B, H, Hkv, N, d, W = 1, 2, 1, 200, 64, 37
    q, k, v = _bf16(22, 1, (B, H, N, d)), _bf16(22, 2, (B, Hkv, N, d)), _bf16(22, 3, (B, Hkv, N, d))
    out = Guarded((B, H, N, d), torch.bfloat16, offset)
    swa.swa_attn_fwd(q, k, v, W, 0.125, out=out.t)
    assert swa.swa_get_device_status() == 0
    assert out.margins_intact()
    assert torch.equal(out.t, swa.swa_attn_fwd(q, k, v, W, 0.125))


@pytest.mark.parametrize("offset", OFFSETS)
def test_varlen_tail_rows_and_margins(swa, offset):
    """Tokens after the last sequence are not written: they keep the sentinel too."""
    H, Hkv, d, W = 4, 2, 128, 64
    cu = [0, 130, 130, 333, 390]
    total = 420  # 30 tokens outside every sequence
    q, k, v = _bf16(23, 1, (total, H, d)), _bf16(23, 2, (total, Hkv, d)), _bf16(23, 3, (total, Hkv, d))
    tcu = torch.tensor(cu, dtype=torch.int64, device="cuda")
    out = Guarded((total, H, d), torch.bfloat16, offset)
    lse = Guarded((H, total), torch.float32, offset)
    swa.swa_attn_varlen(q, k, v, tcu, 203, W, 0.1, n_sink=2, out=out.t, lse=lse.t)
    assert swa.swa_get_device_status() == 0
    assert out.margins_intact() and lse.margins_intact()
    tail = out.raw[out.lo + cu[-1] * H * d * 2:out.hi]
    assert bool(torch.all(tail == SENTINEL)), "rows past the last sequence were written"
    lse_rows = lse.raw[lse.lo:lse.hi].view(H, total * 4)[:, cu[-1] * 4:]
    assert bool(torch.all(lse_rows == SENTINEL)), "lse entries past the last sequence were written"
    ref, ref_lse = swa.swa_attn_varlen(q, k, v, tcu, 203, W, 0.1, n_sink=2, return_lse=True)
    assert torch.equal(out.t[:cu[-1]], ref[:cu[-1]])
    assert torch.equal(lse.t[:, :cu[-1]], ref_lse[:, :cu[-1]])


def _chunk_inputs(seed, B, H, Hkv, Tq, d, W):
    return (_bf16(seed, si.STREAM["q"], (B, H, Tq, d)), _bf16(seed, si.STREAM["k_new"], (B, Hkv, Tq, d)),
            _bf16(seed, si.STREAM["v_new"], (B, Hkv, Tq, d)),
            _bf16(seed, si.STREAM["k_ring"], (B, Hkv, W, d)),
            _bf16(seed, si.STREAM["v_ring"], (B, Hkv, W, d)))


@pytest.mark.parametrize("offset", OFFSETS)
@pytest.mark.parametrize("variant", ["plain", "ragged", "sink"])
def test_chunk_ring_out_lse_and_ring(swa, offset, variant):
    """The ring update writes inside the ring buffers only; out and lse stay in bounds."""
    B, H, Hkv, Tq, d, W = 3, 4, 2, 200, 128, 256
    starts = torch.tensor([1000 + 37, 64, 300], dtype=torch.int64, device="cuda")
    q, kn, vn, rk0, rv0 = _chunk_inputs(24, B, H, Hkv, Tq, d, W)
    out = Guarded((B, H, Tq, d), torch.bfloat16, offset, fill=torch.zeros(()))
    lse = Guarded((B, H, Tq), torch.float32, offset, fill=torch.zeros(()))
    rk = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rk0)
    rv = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rv0)
    kw = {}
    if variant == "sink":
        kw = {"k_sink": _bf16(24, si.STREAM["k_sink"], (B, Hkv, 4, d)),
              "v_sink": _bf16(24, si.STREAM["v_sink"], (B, Hkv, 4, d))}
    lens = torch.tensor([200, 1, 129], dtype=torch.int64, device="cuda")

    def call(o, l, k_ring, v_ring):
        if variant == "ragged":
            swa.swa_attn_chunk_ring_ragged(q, kn, vn, k_ring, v_ring, starts, lens, 0.1,
                                           update_ring=True, out=o, lse=l)
        else:
            swa.swa_attn_chunk_ring(q, kn, vn, k_ring, v_ring, starts, 0.1, update_ring=True,
                                    out=o, lse=l, **kw)
        assert swa.swa_get_device_status() == 0

    call(out.t, lse.t, rk.t, rv.t)
    for g in (out, lse, rk, rv):
        assert g.margins_intact()
    o2, l2 = torch.zeros_like(out.t), torch.zeros_like(lse.t)
    rk2, rv2 = rk0.clone(), rv0.clone()
    call(o2, l2, rk2, rv2)
    assert torch.equal(out.t, o2) and torch.equal(lse.t, l2)
    assert torch.equal(rk.t, rk2) and torch.equal(rv.t, rv2)


@pytest.mark.parametrize("offset", OFFSETS)
@pytest.mark.parametrize("n_sink", [0, 4])
def test_decode_out_lse_and_workspace(swa, offset, n_sink):
    B, H, Hkv, d, W = 5, 8, 2, 128, 640
    q = _bf16(25, si.STREAM["q"], (B, H, d))
    rk, rv = _bf16(25, si.STREAM["k_ring"], (B, Hkv, W, d)), _bf16(25, si.STREAM["v_ring"], (B, Hkv, W, d))
    pos = torch.tensor([5000, 3, 639, 640, 100000], dtype=torch.int64, device="cuda")
    kw = {}
    if n_sink:
        kw = {"k_sink": _bf16(25, si.STREAM["k_sink"], (B, Hkv, n_sink, d)),
              "v_sink": _bf16(25, si.STREAM["v_sink"], (B, Hkv, n_sink, d))}
    need = swa.swa_decode_workspace_bytes(B, H, Hkv, d, W)
    ws = Guarded((need,), torch.uint8, offset, fill=torch.zeros(()))
    out = Guarded((B, H, d), torch.bfloat16, offset)
    lse = Guarded((B, H), torch.float32, offset)
    swa.swa_attn_decode_ring(q, rk, rv, pos, 0.1, workspace=ws.t, out=out.t, lse=lse.t, **kw)
    assert swa.swa_get_device_status() == 0
    for g in (ws, out, lse):
        assert g.margins_intact()
    ref, ref_lse = swa.swa_attn_decode_ring(q, rk, rv, pos, 0.1, return_lse=True, **kw)
    assert torch.equal(out.t, ref) and torch.equal(lse.t, ref_lse)


@pytest.mark.parametrize("offset", OFFSETS)
def test_decode_static_out_and_lse(swa, offset):
    B, H, Hkv, d, W = 3, 4, 4, 64, 300
    q = _bf16(26, si.STREAM["q"], (B, H, d))
    rk, rv = _bf16(26, si.STREAM["k_ring"], (B, Hkv, W, d)), _bf16(26, si.STREAM["v_ring"], (B, Hkv, W, d))
    pos = torch.tensor([299, 7, 12345], dtype=torch.int64, device="cuda")
    out = Guarded((B, H, d), torch.bfloat16, offset)
    lse = Guarded((B, H), torch.float32, offset)
    swa.swa_attn_decode_ring_static(q, rk, rv, pos, 0.1, out=out.t, lse=lse.t)
    assert swa.swa_get_device_status() == 0
    assert out.margins_intact() and lse.margins_intact()
    ref, ref_lse = swa.swa_attn_decode_ring(q, rk, rv, pos, 0.1, return_lse=True)
    assert torch.equal(out.t, ref) and torch.equal(lse.t, ref_lse)


@pytest.mark.parametrize("offset", OFFSETS)
def test_backward_gradients_and_workspace(swa, offset):
    B, H, Hkv, N, d, W = 1, 4, 2, 300, 128, 100
    q, k, v = _bf16(27, 1, (B, H, N, d)), _bf16(27, 2, (B, Hkv, N, d)), _bf16(27, 3, (B, Hkv, N, d))
    dout = _bf16(27, si.STREAM["extra"], (B, H, N, d))
    o, lse = swa.swa_attn_fwd(q, k, v, W, 0.1, return_lse=True)
    need = int(swa.lib().swa_attn_bwd_workspace_bytes(B, H, N))
    ws = Guarded((need,), torch.uint8, offset, fill=torch.zeros(()))
    dq = Guarded((B, H, N, d), torch.bfloat16, offset)
    dk = Guarded((B, Hkv, N, d), torch.bfloat16, offset)
    dv = Guarded((B, Hkv, N, d), torch.bfloat16, offset)
    swa.swa_attn_bwd(q, k, v, o, dout, lse, W, 0.1, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    assert swa.swa_get_device_status() == 0
    for g in (ws, dq, dk, dv):
        assert g.margins_intact()
    rq, rk, rv = swa.swa_attn_bwd(q, k, v, o, dout, lse, W, 0.1)
    assert torch.equal(dq.t, rq) and torch.equal(dk.t, rk) and torch.equal(dv.t, rv)


@pytest.mark.parametrize("offset", OFFSETS)
def test_metadata_and_slot_positions(swa, offset):
    B, n_q, W = 3, 300, 200
    q_pos0 = torch.tensor([0, 1000 + 5, 77], dtype=torch.int64, device="cuda")
    nqt = math.ceil(n_q / 64)
    nkt = math.ceil(W / 32) + math.ceil(n_q / 32)
    cls = Guarded((B, nqt, nkt), torch.int8, offset)
    rng = Guarded((B, nqt, 4), torch.int32, offset)
    swa.swa_block_meta(1, n_q, 0, W, 64, 32, q_pos0=q_pos0, classes=cls.t, ranges=rng.t)
    assert cls.margins_intact() and rng.margins_intact()
    c2, r2 = swa.swa_block_meta(1, n_q, 0, W, 64, 32, q_pos0=q_pos0)
    assert torch.equal(cls.t, c2) and torch.equal(rng.t, r2)
    sp = Guarded((B, W), torch.int64, offset)
    swa.swa_ring_slot_positions(q_pos0, W, out=sp.t)
    assert sp.margins_intact()
    assert torch.equal(sp.t, swa.swa_ring_slot_positions(q_pos0, W))


@pytest.mark.parametrize("offset", OFFSETS)
def test_ring_write_stays_in_ring(swa, offset):
    B, Hkv, T, d, W = 3, 2, 70, 64, 32
    kn, vn = _bf16(28, 6, (B, Hkv, T, d)), _bf16(28, 7, (B, Hkv, T, d))
    rk0, rv0 = _bf16(28, 4, (B, Hkv, W, d)), _bf16(28, 5, (B, Hkv, W, d))
    starts = torch.tensor([0, 31, 1000], dtype=torch.int64, device="cuda")
    rk = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rk0)
    rv = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rv0)
    swa.swa_ring_write(kn, vn, rk.t, rv.t, starts)
    assert rk.margins_intact() and rv.margins_intact()
    rk2, rv2 = rk0.clone(), rv0.clone()
    swa.swa_ring_write(kn, vn, rk2, rv2, starts)
    assert torch.equal(rk.t, rk2) and torch.equal(rv.t, rv2)


@pytest.mark.parametrize("offset", [0, 256])
def test_chunk_split_out_lse_workspace_and_ring(swa, offset):
    """The split chunk call writes inside out, lse, the ring and its workspace only."""
    B, H, Hkv, Tq, d, W = 3, 4, 2, 200, 128, 256
    starts = torch.tensor([1000 + 37, 64, 300], dtype=torch.int64, device="cuda")
    lens = torch.tensor([200, 1, 129], dtype=torch.int64, device="cuda")
    q, kn, vn, rk0, rv0 = _chunk_inputs(29, B, H, Hkv, Tq, d, W)
    need = swa.swa_chunk_split_workspace_bytes(B, H, Hkv, Tq, d, W)
    ws = Guarded((need,), torch.uint8, offset, fill=torch.zeros(()))
    out = Guarded((B, H, Tq, d), torch.bfloat16, offset, fill=torch.zeros(()))
    lse = Guarded((B, H, Tq), torch.float32, offset, fill=torch.zeros(()))
    rk = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rk0)
    rv = Guarded((B, Hkv, W, d), torch.bfloat16, offset, fill=rv0)
    swa.swa_attn_chunk_ring_split(q, kn, vn, rk.t, rv.t, starts, 0.1, chunk_len=lens,
                                  update_ring=True, out=out.t, lse=lse.t, workspace=ws.t)
    assert swa.swa_get_device_status() == 0
    for g in (ws, out, lse, rk, rv):
        assert g.margins_intact()
