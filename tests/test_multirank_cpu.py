"""Host logic of a multi-rank bench run, on CPU ranks with the gloo backend (world size 2):
the job time is the slowest rank's, and the job throughput counts every rank's units."""
import os
import socket
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 10 + r ms for the step and 3 - r ms for e2e
        step, e2e = bench.max_over_ranks([10.0 + rank, 3.0 - rank], torch.device("cpu"))
        value = bench.job_throughput(world, 1000.0, step)
        dist.barrier()
        out[rank] = (step, e2e, value)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo_world2():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        step, e2e, value = out[r]
        assert step == 11.0 and e2e == 3.0
        assert value == pytest.approx(world * 1000.0 / 11e-3)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.5, 2.5], torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_throughput(1, 10.0, 2.0) == pytest.approx(5000.0)
