"""The multi-rank host logic of bench.py on two gloo ranks (CPU, no GPU).

Each rank runs its own batch (weak scaling, no data-path collective); the only
collectives are the barrier and the max over ranks of the timing, so that
`value` = every rank's work / the slowest rank's time.
"""

import os
import socket
import subprocess
import sys
from datetime import timedelta

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    import bench
    import swa_inputs as si
    from swa_inputs.workloads import WORKLOADS

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = 1.0 + rank  # rank 1 is the slow one
        job_ms = bench.max_over_ranks(ms, world, "cpu")
        dist.barrier()
        w = WORKLOADS["tiny"]
        seed = w.seed + bench.rank_seed_offset(rank)
        q = si.normal_bf16(seed, si.STREAM["q"], (1, 2, 8, 4))
        np.save(os.path.join(out_dir, f"q{rank}.npy"), q)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(f"{job_ms} {bench.job_rate(1e12, world, job_ms, 1e12)}")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.spawn(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True)
    res = [open(tmp_path / f"r{r}.txt").read().split() for r in range(world)]
    for job_ms, rate in res:
        assert float(job_ms) == 2.0              # both ranks see the slowest time
        assert float(rate) == 1e12 * 2 / 2e-3 / 1e12  # whole-job work over that time
    q0, q1 = np.load(tmp_path / "q0.npy"), np.load(tmp_path / "q1.npy")
    assert not np.array_equal(q0, q1)             # independent batches per rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_rate(2e12, 1, 2.0, 1e12) == 1000.0


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "3", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
