"""Multi-process checks of the benchmark's rank logic on CPU (gloo, world
size 2): the timed region is the maximum over ranks, the whole-job value sums
the ranks' work over that time, and the reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cpu = torch.device("cpu")
        bench.barrier(cpu)
        secs = 1.0 + 0.5 * rank                      # rank 1 is the slower one
        worst = bench.max_over_ranks(secs, cpu)
        value = bench.whole_job_gbs(4e9, 10, world, worst)
        ref = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), rank, world) if rank else None
        out[rank] = (bench.dist_env(), worst, value, ref)
    finally:
        dist.destroy_process_group()


def test_rank_reduction_and_whole_job_value():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        env, worst, value, ref = res[rank]
        assert env == (rank, rank, world)
        assert worst == pytest.approx(1.5)                      # max over ranks, not the local time
        assert value == pytest.approx(4e9 * 10 * world / 1.5 / 1e9)
    assert res[1][3] is None                                    # the reference arm does no work off rank 0


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25
    assert bench.whole_job_gbs(1e9, 2, 1, 1.0) == pytest.approx(2.0)
