"""The N > 1 path of bench.py on CPU: two gloo ranks, as torchrun launches them.

The virtual ranks of one problem all run on one GPU, so several GPUs run independent replicas
(weak scaling) and the only cross-rank step is the timing: the job's time is the slowest
replica's, and its throughput counts every replica's work.  The reference arm prints from
rank 0 only; other ranks exit 0 without work."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]          # rank 1 is the slow replica
        m = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        v = bench.whole_job_tflops(1e14, 5, world, m)
        dist.barrier()
        out[rank] = (m, v)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_value_gloo():
    port = 29500 + os.getpid() % 2000
    with mp.get_context("spawn").Manager() as man:
        out = man.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for r in (0, 1):
        m, v = res[r]
        assert m == 150.0                     # the slowest replica's time on every rank
        assert v == pytest.approx(2 * 1e14 * 5 / 0.150 / 1e12)


def test_single_rank_is_the_local_time():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    assert bench.max_over_ranks(12.5, 1, torch.device("cpu")) == 12.5
    assert bench.whole_job_tflops(2e12, 3, 1, 1000.0) == pytest.approx(6.0)


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
