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


def _shard_main(rank, world, port, out):
    """Each rank quantizes its own rows of one weight (oracle, on the CPU) and computes its
    output slice; the slices are joined by an all_gather."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import numpy as np
    import oracle
    from bit_gemm_wise_b200 import shard, synth
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        N, K, g = 300, 256, 64
        W = synth.bf16_bits(synth.student_t3_weight(N, K, 0, 61))
        x = synth.bf16_bits(synth.normal((2, K), 1.0, 0, 62))
        n0, n1 = shard.column_shard(N, world, rank)
        codes, scales, zeros, _ = oracle.quantize(W[n0:n1], g, "asym", synth.clip_grid_20(), want_chosen=False)
        y = oracle.gemv_ref(x, codes, scales, zeros, g, "asym")
        parts = [None] * world
        dist.all_gather_object(parts, (n0, n1, codes, scales, zeros, y))
        out[rank] = parts
    finally:
        dist.destroy_process_group()


def test_column_parallel_split_gloo_world2():
    """Two gloo ranks each own whole 128-row weight tiles of W[300, 256]; the gathered codes,
    scales, zero points and outputs equal those of the unsplit layer exactly."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import oracle
    from bit_gemm_wise_b200 import synth
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    N, K, g = 300, 256, 64
    W = synth.bf16_bits(synth.student_t3_weight(N, K, 0, 61))
    x = synth.bf16_bits(synth.normal((2, K), 1.0, 0, 62))
    codes, scales, zeros, _ = oracle.quantize(W, g, "asym", synth.clip_grid_20(), want_chosen=False)
    y = oracle.gemv_ref(x, codes, scales, zeros, g, "asym")
    for r in range(world):
        parts = out[r]
        assert [(p[0], p[1]) for p in parts] == [(0, 128), (128, 300)]
        assert np.array_equal(np.concatenate([p[2] for p in parts]), codes)
        assert np.array_equal(np.concatenate([p[3] for p in parts]), scales)
        assert np.array_equal(np.concatenate([p[4] for p in parts]), zeros)
        assert np.array_equal(np.concatenate([p[5] for p in parts], axis=1), y)


def test_column_shard_covers_every_row_once():
    sys.path.insert(0, ROOT)
    from bit_gemm_wise_b200 import shard
    for N in (0, 1, 127, 128, 300, 3840, 15360, 14336, 5760):
        for world in (1, 2, 3, 4, 8):
            for granule in (1, 128):
                spans = [shard.column_shard(N, world, r, granule) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == N
                for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                    assert a1 == b0 and a0 <= a1
                # whole granules except at the end of W; sizes differ by at most one granule
                assert all(a0 % granule == 0 for a0, _ in spans)
                units = [(-(-a1 // granule)) - a0 // granule for a0, a1 in spans]
                assert max(units) - min(units) <= 1
    with pytest.raises(ValueError):
        shard.column_shard(100, 2, 2)
