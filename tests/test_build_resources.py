"""Compiler resource report of the CUDA library (CPU, needs nvcc).

The forward attention kernel re-splits its registers between warp groups
(setmaxnreg), a split written for exactly 168 registers per thread at launch
with 384 threads; the library also refuses to launch it otherwise.  This
test compiles the library with ptxas' resource report and checks, before
any GPU run, that every instantiation of the forward kernel gets exactly
that launch count, that the linear and packed-varlen instantiations at
d = 128 do not spill, and that the backward kernels stay within the 255
registers of a 192-thread block.
"""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "sliding_window_sparse_b200", "csrc")
NVCC = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"

pytestmark = pytest.mark.skipif(not os.path.exists(NVCC), reason="nvcc not available")


def _fwd2_launch_regs():
    text = open(os.path.join(CSRC, "swa_fwd2.cuh")).read()
    return int(re.search(r"constexpr int kFwd2LaunchRegs = (\d+);", text).group(1))


@pytest.fixture(scope="module")
def report(tmp_path_factory):
    out = tmp_path_factory.mktemp("ptxas") / "libswa_check.so"
    cmd = [NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v", "-o", str(out),
           os.path.join(CSRC, "swa_lib.cu")]
    res = subprocess.run(cmd, capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-2000:]
    kernels, name = {}, None
    for line in res.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            name = m.group(1)
            kernels[name] = {}
            continue
        if name is None:
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m:
            kernels[name]["spill"] = int(m.group(1)) + int(m.group(2))
        m = re.search(r"Used (\d+) registers", line)
        if m:
            kernels[name]["regs"] = int(m.group(1))
    return kernels


def _fwd2(report):
    """{(D, MODE, SINK): resources} for every forward instantiation."""
    out = {}
    for name, r in report.items():
        m = re.search(r"fwd2_kernelILi(\d+)ELi(\d)ELb(\d)E", name)
        if m:
            out[(int(m.group(1)), int(m.group(2)), bool(int(m.group(3))))] = r
    return out


def test_every_forward_instantiation_gets_the_split_launch_count(report):
    fwd = _fwd2(report)
    assert len(fwd) == 12          # D in {64, 128} x MODE in {0, 1, 2} x SINK
    want = _fwd2_launch_regs()
    for key, r in fwd.items():
        assert r.get("regs") == want, (key, r)


def test_headline_forward_kernels_do_not_spill(report):
    fwd = _fwd2(report)
    for key in ((128, 0, False), (128, 2, False), (128, 0, True), (128, 2, True)):
        assert fwd[key].get("spill", 0) == 0, (key, fwd[key])


def test_backward_kernels_fit_their_block(report):
    bwd = {n: r for n, r in report.items() if "bwd_dq_kernel" in n or "bwd_dkdv_kernel" in n}
    assert len(bwd) == 16          # 2 kernels x D in {64, 128} x layout {0, 2} x SINK
    for name, r in bwd.items():
        assert r.get("regs", 0) <= 255, (name, r)


def test_ring_layout_forward_spills_stay_small(report):
    """The ring-layout (chunk) instantiations carry the split call's item list and
    part bookkeeping; their spills stay a few words (16-20 bytes of stores plus
    as many of loads when this was written), far from the softmax's score row."""
    fwd = _fwd2(report)
    for key, r in fwd.items():
        if key[1] == 1:
            assert r.get("spill", 0) <= 64, (key, r)  # spill stores + spill loads


def test_split_chunk_kernels_are_built(report):
    """The split chunk call's schedule and merge kernels exist for d = 64 and 128."""
    for kern in ("chunk_split_schedule_kernel", "chunk_split_merge_kernel"):
        found = [n for n in report if kern in n]
        assert len(found) == 2, (kern, found)
