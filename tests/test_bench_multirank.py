"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): the
job's time is the slowest rank's, throughput counts every rank's work, and
the reference arm runs on rank 0 alone."""
import importlib.util
import os
import subprocess
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        b.barrier(dist)
        local_ms = [100.0, 150.0][rank]  # rank 1 is the slow one
        ms_step, gbs = b.job_throughput(local_ms, 10, 1e9, dist, world)
        out[rank] = (b.max_over_ranks(float(rank), dist), ms_step, gbs)
        b.barrier(dist)
    finally:
        dist.destroy_process_group()


def test_job_throughput_two_ranks_gloo():
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank, args=(2, 29531, out), nprocs=2, join=True)
    for r in (0, 1):
        mx, ms_step, gbs = out[r]
        assert mx == 1.0
        assert abs(ms_step - 15.0) < 1e-9                     # slowest rank: 150 ms / 10 steps
        assert abs(gbs - 2 * 1e9 / 15e-3 / 1e9) < 1e-6        # both ranks' bytes


def test_reference_arm_nonzero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
