"""Failure detection on the device: a bounded wait that runs out.

Every mbarrier wait of the attention kernels gives up after a time limit,
records a timeout in the device status word and raises its CTA's abort flag,
so that a broken handshake ends the kernel instead of hanging the GPU.  The
real kernels are never made to time out here: swa_selftest_wait runs the same
wait code in a one-CTA kernel with one barrier nobody arrives at (no copies, no
tensor memory) and a short limit, then returns.  These tests check that the
wait gives up, that the other waiters follow through the abort flag instead of
waiting out their own limit, that the host reads SWA_ERR_TIMEOUT, that reading
clears it, and that the context stays usable afterwards.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import swa_inputs as si
from tests._util import assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

SWA_OK = 0
SWA_ERR_INVALID_ARG = 1
SWA_ERR_TIMEOUT = 5


@pytest.fixture(scope="module")
def swa(cuda_ok):
    import sliding_window_sparse_b200 as m

    return m


def _selftest(swa, limit_ns, arrive):
    res = torch.full((5,), -1, dtype=torch.int32, device="cuda")
    st = swa.lib().swa_selftest_wait(limit_ns, arrive, res.data_ptr(),
                                     torch.cuda.current_stream().cuda_stream)
    assert st == SWA_OK
    status = swa.swa_get_device_status()
    return status, res.cpu().numpy()


def test_wait_that_nobody_ends_times_out(swa):
    assert swa.swa_get_device_status() == SWA_OK
    limit_ns = 20_000_000  # 20 ms
    status, res = _selftest(swa, limit_ns, arrive=0)
    assert status == SWA_ERR_TIMEOUT
    assert list(res[:4]) == [0, 0, 0, 0], res
    # the first waiter gave up after its own limit; the other 96 lanes followed
    # through the abort flag, not after their own 1 s limit
    assert limit_ns / 1000 <= res[4] < limit_ns / 1000 + 200_000, res[4]
    # reading the status cleared it
    assert swa.swa_get_device_status() == SWA_OK


def test_wait_that_is_ended_succeeds(swa):
    status, res = _selftest(swa, 20_000_000, arrive=1)
    assert status == SWA_OK
    assert list(res[:4]) == [1, 32, 32, 32], res
    assert res[4] < 20_000


def test_context_usable_after_a_timeout(swa):
    """A timed-out self-test leaves the device usable: a prefill afterwards is correct."""
    status, _ = _selftest(swa, 1_000_000, arrive=0)
    assert status == SWA_ERR_TIMEOUT
    B, H, Hkv, N, d, W = 1, 2, 1, 200, 128, 50
    q = si.normal_bf16(31, 1, (B, H, N, d))
    k = si.normal_bf16(31, 2, (B, Hkv, N, d))
    v = si.normal_bf16(31, 3, (B, Hkv, N, d))
    out = swa.swa_attn_fwd(to_dev(q), to_dev(k), to_dev(v), W, 1 / math.sqrt(d))
    assert swa.swa_get_device_status() == SWA_OK
    assert_close(to_f64(out), oracle.swa_forward(q, k, v, W, 1 / math.sqrt(d)), what="after")


def test_selftest_rejects_bad_limits(swa):
    res = torch.zeros(5, dtype=torch.int32, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert swa.lib().swa_selftest_wait(10, 0, res.data_ptr(), s) == SWA_ERR_INVALID_ARG
    assert swa.lib().swa_selftest_wait(2_000_000_000, 0, res.data_ptr(), s) == SWA_ERR_INVALID_ARG
    assert swa.lib().swa_selftest_wait(1_000_000, 0, None, s) == SWA_ERR_INVALID_ARG
    assert np.all(res.cpu().numpy() == 0)
