"""swa_attn_decode_ring_static: decode for callers that cannot provide scratch.

Some callers have no device allocator to hand the library a workspace (a
plugin or foreign-language host that owns none, or a process that reserved all
free device memory up front).  The static entry point keeps its split
partials in a fixed 16 MiB device array inside the library instead.  These
tests call it through the C ABI and check it against the workspace entry point
on two calls in a row, with different inputs, so that contents left in the
shared array by the first call cannot leak into the second.

This file is named to be collected last; it depends on no state from the
other tests and also passes alone in a fresh process.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

import swa_inputs as si
from tests._util import MAX_ABS, MEAN_ABS, assert_close, to_dev, to_f64

pytestmark = pytest.mark.gpu

STATIC_SCRATCH_BYTES = 16 << 20


@pytest.fixture(scope="module")
def lib(cuda_ok):
    from sliding_window_sparse_b200 import _native

    return _native.lib()


def _inputs(seed, B, H, Hkv, d, W, pos):
    q = to_dev(si.normal_bf16(seed, si.STREAM["q"], (B, H, d)))
    rk = to_dev(si.normal_bf16(seed, si.STREAM["k_ring"], (B, Hkv, W, d)))
    rv = to_dev(si.normal_bf16(seed, si.STREAM["v_ring"], (B, Hkv, W, d)))
    p = torch.tensor(pos, dtype=torch.int64, device="cuda")
    return q, rk, rv, p


def _call_static(lib, q, rk, rv, p, W, scale):
    B, H, d = q.shape
    Hkv = rk.shape[1]
    out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    st = lib.swa_attn_decode_ring_static(q.data_ptr(), rk.data_ptr(), rv.data_ptr(), p.data_ptr(),
                                         out.data_ptr(), lse.data_ptr(), B, H, Hkv, d, W, scale,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.swa_status_string(st)
    return out, lse


def _call_workspace(lib, q, rk, rv, p, W, scale):
    B, H, d = q.shape
    Hkv = rk.shape[1]
    need = lib.swa_decode_workspace_bytes(B, H, Hkv, d, W)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    st = lib.swa_attn_decode_ring(q.data_ptr(), rk.data_ptr(), rv.data_ptr(), p.data_ptr(),
                                  out.data_ptr(), lse.data_ptr(), B, H, Hkv, d, W, scale,
                                  ws.data_ptr(), need, torch.cuda.current_stream().cuda_stream)
    assert st == 0, lib.swa_status_string(st)
    return out, lse


@pytest.mark.parametrize("B,H,Hkv,d,W,pos_a,pos_b", [
    (64, 32, 8, 128, 4096, None, None),          # the decode workload's shape, full windows
    (3, 8, 2, 64, 300, [5, 299, 1000], [70, 0, 4000]),
])
def test_static_matches_workspace_twice(lib, B, H, Hkv, d, W, pos_a, pos_b):
    scale = 1.0 / math.sqrt(d)
    if pos_a is None:
        pos_a = list(si.uniform_int(4, si.STREAM["ctx_len"], B, 4096, 131072) - 1)
        pos_b = list(si.uniform_int(5, si.STREAM["ctx_len"], B, 4096, 131072) - 1)
    for call, (seed, pos) in enumerate([(40, pos_a), (41, pos_b)]):
        q, rk, rv, p = _inputs(seed, B, H, Hkv, d, W, pos)
        got, got_lse = _call_static(lib, q, rk, rv, p, W, scale)
        ref, ref_lse = _call_workspace(lib, q, rk, rv, p, W, scale)
        torch.cuda.synchronize()
        assert lib.swa_get_device_status(None) == 0
        assert_close(to_f64(got), to_f64(ref), MAX_ABS, MEAN_ABS, what=f"call {call}")
        assert np.max(np.abs(to_f64(got_lse) - to_f64(ref_lse))) < 1e-3


def test_static_rejects_requests_beyond_its_array(lib):
    # B=64, H=512, Hkv=64, d=128, W=4096 needs far more than 16 MiB of partials
    B, H, Hkv, d, W = 64, 512, 64, 128, 4096
    assert lib.swa_decode_workspace_bytes(B, H, Hkv, d, W) > STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x100000)  # never dereferenced: rejected before any launch
    st = lib.swa_attn_decode_ring_static(fake, fake, fake, fake, fake, None, B, H, Hkv, d, W,
                                         0.1, None)
    assert st == 4  # SWA_ERR_WORKSPACE
