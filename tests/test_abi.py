"""The C-ABI library loads, exports every symbol include/swa.h declares, and
rejects bad arguments before touching the GPU.  No compute call is made."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "swa.h")


@pytest.fixture(scope="module")
def native():
    from sliding_window_sparse_b200 import build

    build.build()
    from sliding_window_sparse_b200 import _native

    return _native


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SWA_API\s+[\w\s\*]*?\b(swa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for want in ["swa_block_meta", "swa_attn_fwd", "swa_attn_bwd", "swa_attn_chunk_ring",
                 "swa_attn_chunk_ring_ragged", "swa_attn_decode_ring",
                 "swa_decode_workspace_bytes", "swa_ring_write", "swa_ring_slot_positions",
                 "swa_get_device_status", "swa_status_string", "swa_version"]:
        assert want in names


def test_header_is_plain_c(tmp_path):
    """The boundary header compiles as strict C99 and links against the library:
    plain pointers and sizes, no C++ or torch types."""
    import shutil
    import subprocess

    if not shutil.which("gcc"):
        pytest.skip("no C compiler")
    src = tmp_path / "use_header.c"
    src.write_text('#include "swa.h"\n'
                   "int main(void) { return swa_version() > 0 && "
                   "swa_status_string(0) != 0 ? 0 : 1; }\n")
    from sliding_window_sparse_b200 import build

    lib = build.build()
    exe = tmp_path / "use_header"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe), str(lib),
                    "-Wl,-rpath," + os.path.dirname(str(lib))], check=True)
    assert subprocess.run([str(exe)]).returncode == 0


def test_every_declared_symbol_is_exported(native):
    lib = native.lib()
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in native.SIGNATURES, f"{name} has no ctypes signature"


def test_only_declared_symbols_are_exported(native):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", native.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted({line.split()[-1] for line in out.splitlines()
                       if line.split()[-2] in ("T", "t") and line.split()[-1].startswith("swa_")})
    assert exported == declared_symbols()


def test_status_strings(native):
    lib = native.lib()
    assert lib.swa_status_string(0) == b"SWA_OK"
    assert lib.swa_status_string(1) == b"SWA_ERR_INVALID_ARG"
    assert lib.swa_status_string(4) == b"SWA_ERR_WORKSPACE"
    assert lib.swa_status_string(99) == b"SWA_ERR_UNKNOWN"
    assert lib.swa_version() >> 16 == 1


def test_workspace_size_host_only(native):
    lib = native.lib()
    n = lib.swa_decode_workspace_bytes(64, 32, 8, 128, 4096)
    assert n >= 64 * 32 * 128 * 4  # at least one fp32 partial per (b, h)
    assert lib.swa_decode_workspace_bytes(0, 32, 8, 128, 4096) == 0
    # more splits for small batches: still a multiple of 256 bytes per region
    assert lib.swa_decode_workspace_bytes(1, 8, 1, 64, 4096) % 256 == 0


FAKE = ctypes.c_void_p(0x100000)  # aligned non-null address: never dereferenced


@pytest.mark.parametrize("args,code", [
    # (B, H, Hkv, N, d, W, scale)
    ((1, 4, 4, 128, 96, 16, 0.1), 2),      # unsupported head dim
    ((1, 4, 3, 128, 64, 16, 0.1), 1),      # H % Hkv != 0
    ((0, 4, 4, 128, 64, 16, 0.1), 1),      # B < 1
    ((1, 4, 4, 128, 64, 0, 0.1), 1),       # W < 1
    ((1, 4, 4, 128, 64, -5, 0.1), 1),      # negative window
    ((1, 4, 4, 128, 64, 16, 0.0), 1),      # scale <= 0
    ((1, 4, 4, 128, 64, 16, float("nan")), 1),
    ((1, 4, 4, 0, 64, 16, 0.1), 1),        # N < 1
])
def test_fwd_rejects_bad_arguments(native, args, code):
    B, H, Hkv, N, d, W, scale = args
    st = native.lib().swa_attn_fwd(FAKE, FAKE, FAKE, FAKE, None, B, H, Hkv, N, d, W, scale, None)
    assert st == code


def test_fwd_rejects_null_and_misaligned(native):
    lib = native.lib()
    assert lib.swa_attn_fwd(None, FAKE, FAKE, FAKE, None, 1, 4, 4, 128, 64, 16, 0.1, None) == 1
    odd = ctypes.c_void_p(0x100008)
    assert lib.swa_attn_fwd(odd, FAKE, FAKE, FAKE, None, 1, 4, 4, 128, 64, 16, 0.1, None) == 1


def test_ragged_chunk_rejects_null_lengths(native):
    lib = native.lib()
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert lib.swa_attn_chunk_ring_ragged(*args, None, FAKE, None, 1, 4, 4, 128, 64, 64, 0.1, 0,
                                          None) == 1
    assert lib.swa_attn_chunk_ring_ragged(*args, FAKE, FAKE, None, 1, 4, 4, 0, 64, 64, 0.1, 0,
                                          None) == 1


def test_decode_rejects_small_workspace(native):
    lib = native.lib()
    need = lib.swa_decode_workspace_bytes(2, 8, 2, 128, 256)
    st = lib.swa_attn_decode_ring(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 128, 256, 0.1,
                                  FAKE, need - 1, None)
    assert st == 4
    st = lib.swa_attn_decode_ring(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 8, 2, 128, 256, 0.1,
                                  None, need, None)
    assert st == 4


def test_chunk_and_meta_reject_bad_arguments(native):
    lib = native.lib()
    # chunk: null q_start, W too large
    assert lib.swa_attn_chunk_ring(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, 1, 4, 4, 64,
                                   64, 128, 0.1, 0, None) == 1
    assert lib.swa_attn_chunk_ring(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 4, 4, 64,
                                   64, 1 << 30, 0.1, 0, None) == 1
    # meta: bad mode, bad tile, ring mode without start positions, no outputs
    assert lib.swa_block_meta(2, 1, 8, 8, None, 3, 2, 2, FAKE, FAKE, None) == 1
    assert lib.swa_block_meta(0, 1, 8, 8, None, 3, 0, 2, FAKE, FAKE, None) == 1
    assert lib.swa_block_meta(1, 1, 8, 8, None, 3, 2, 2, FAKE, FAKE, None) == 1
    assert lib.swa_block_meta(0, 1, 8, 8, None, 3, 2, 2, None, None, None) == 1
    # ring write / slot positions
    assert lib.swa_ring_write(FAKE, FAKE, FAKE, FAKE, None, 1, 1, 4, 64, 8, None) == 1
    assert lib.swa_ring_slot_positions(1, None, 8, FAKE, None) == 1


def test_product_package_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "sliding_window_sparse_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f"{f} mentions the oracle"
