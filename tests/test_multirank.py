"""The N > 1 host path of bench.py on CPU: two gloo ranks.

Each rank runs its own replica (the pass has no cross-sequence exchange), so
the only collective steps are the barrier and the max over ranks of the
timings; the job's value is all ranks' tokens over the slowest rank's time.
The reference arm prints from rank 0 only; other ranks exit 0 without work.
"""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, per_rank_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        t = torch.tensor(per_rank_ms[rank], dtype=torch.float64)
        agg = bench.max_over_ranks(t, world).tolist()
        value = bench.job_throughput(world, 8192, 10, agg[0])
        out[rank] = (agg, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    world = 2
    per_rank_ms = [[5.0, 1.0, 9.0], [7.5, 0.5, 9.5]]
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), per_rank_ms, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    for rank in range(world):
        agg, value = res[rank]
        assert agg == [7.5, 1.0, 9.5]          # element-wise max over the ranks
        # both ranks' tokens over the slowest rank's time
        assert value == pytest.approx(2 * 8192 * 10 / 7.5e-3)


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    t = torch.tensor([3.0, 4.0], dtype=torch.float64)
    assert bench.max_over_ranks(t, 1).tolist() == [3.0, 4.0]
    assert bench.job_throughput(1, 100, 4, 2.0) == pytest.approx(100 * 4 / 2e-3)


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
