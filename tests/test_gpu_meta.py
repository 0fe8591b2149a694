"""Device-built tile metadata and ring-slot map: bit-exact against the oracle."""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


LINEAR_CASES = [
    # (B, n, W, tile_q, tile_k, q_pos0)
    (1, 8, 3, 2, 2, None),          # M003 note section 04 worked example
    (1, 8, 3, 4, 4, None),
    (1, 512, 64, 64, 64, None),     # tiny workload, 64x64 tiles
    (1, 8192, 4096, 128, 128, None),  # Mistral-shaped prefill
    (2, 32768, 512, 128, 128, None),  # narrow window
    (1, 1000, 130, 128, 64, None),  # ragged tails
    (3, 300, 7, 16, 32, [0, 5, 1000]),
    (1, 77, 500, 16, 32, None),     # W >= N: full causal
    (1, 129, 1, 128, 128, None),    # W = 1
]


@pytest.mark.parametrize("B,n,W,tq,tk,qp", LINEAR_CASES)
def test_block_meta_linear_bit_exact(swa, B, n, W, tq, tk, qp):
    q_pos0 = None if qp is None else torch.tensor(qp, dtype=torch.int64, device="cuda")
    cls, rng = swa.swa_block_meta(0, n, n, W, tq, tk, q_pos0=q_pos0, B=B)
    ref_c, ref_r = oracle.tile_classes(0, B, n, n, W, tq, tk, q_pos0=qp)
    assert np.array_equal(cls.cpu().numpy(), ref_c)
    assert np.array_equal(rng.cpu().numpy(), ref_r)


def test_block_meta_worked_example_counts(swa):
    for tile, live, coords in [(2, 7, 28), (4, 3, 48)]:
        cls, _ = swa.swa_block_meta(0, 8, 8, 3, tile, tile, B=1)
        n_live = int((cls.cpu().numpy() != 0).sum())
        assert n_live == live and n_live * tile * tile == coords


RING_CASES = [
    # (W, Tq, q_starts, tile_q, tile_k)
    (4096, 512, [12288] * 4, 128, 128),           # chunk workload (ring-aligned)
    (4096, 512, [12288 + 37, 5000, 4095, 4096], 128, 128),  # unaligned starts / wrap
    (64, 40, [100, 10, 0, 64], 16, 16),           # partly empty ring, zero start
    (48, 100, [1000, 47], 32, 32),                 # chunk longer than the ring
    (300, 129, [301, 7], 128, 128),               # ragged ring tiles
]


@pytest.mark.parametrize("W,Tq,qs,tq,tk", RING_CASES)
def test_block_meta_ring_bit_exact(swa, W, Tq, qs, tq, tk):
    q_pos0 = torch.tensor(qs, dtype=torch.int64, device="cuda")
    cls, rng = swa.swa_block_meta(1, Tq, 0, W, tq, tk, q_pos0=q_pos0)
    ref_c, ref_r = oracle.tile_classes(1, len(qs), Tq, 0, W, tq, tk, q_pos0=qs)
    assert np.array_equal(cls.cpu().numpy(), ref_c)
    assert np.array_equal(rng.cpu().numpy(), ref_r)


@pytest.mark.parametrize("W", [1, 3, 64, 4096, 1000])
def test_ring_slot_positions_bit_exact(swa, W):
    ns = [0, 1, W - 1, W, W + 1, 3 * W + 5, 12288, 131071, 7]
    n_written = torch.tensor(ns, dtype=torch.int64, device="cuda")
    got = swa.swa_ring_slot_positions(n_written, W).cpu().numpy()
    for i, n in enumerate(ns):
        assert np.array_equal(got[i], oracle.ring_positions(max(n, 0), W))


def test_negative_start_sets_device_status(swa):
    q_pos0 = torch.tensor([-3], dtype=torch.int64, device="cuda")
    swa.swa_block_meta(1, 16, 0, 8, 16, 16, q_pos0=q_pos0)
    assert swa.swa_get_device_status() == 6
    assert swa.swa_get_device_status() == 0  # cleared
