"""CPU: the benchmark's multi-rank aggregation, with two gloo ranks.

bench.py times every rank's own replica and reports the slowest rank's time over the
calls of all ranks; these checks run that host logic (max_over_ranks,
job_us_per_call) in two processes on the CPU, no GPU involved."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" (10 + 5 r) ms for its steps and (20 - r) ms end to end
        ms, ms_e2e = bench.max_over_ranks([10.0 + 5.0 * rank, 20.0 - rank])
        out[rank] = (ms, ms_e2e, bench.job_us_per_call(ms, 1000, world))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        ms, ms_e2e, us = out[r]
        assert ms == 15.0 and ms_e2e == 20.0          # the slowest rank's time, on every rank
        assert us == pytest.approx(15.0 * 1000.0 / (1000 * world))   # 7.5 us per call for the job


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.5]) == [3.0, 4.5]
    assert bench.job_us_per_call(26.0, 1000, 1) == pytest.approx(26.0)
