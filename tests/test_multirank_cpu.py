"""The N > 1 path of bench.py on CPU: two gloo ranks (world size 2).

bench.py runs one replica of the step per GPU (the path needs no data-path
collective); its only collectives are the barriers around the timed region
and the max over ranks of the step time.  These tests run those host-side
pieces as two real processes over gloo on 127.0.0.1.
"""
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


def _rank_main(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        ms = bench.max_over_ranks(local_ms[rank], dist, torch.device("cpu"))
        value = bench.job_value(world, ms)
        # the reference arm does its work on rank 0 only; other ranks return at once
        class A:
            steps, warmup, gpus = 1, 0, world
        skipped = rank != 0 and bench.run_reference(A, rank) is None
        dist.barrier()
        out[rank] = (ms, value, skipped)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_step():
    world = 2
    local_ms = [0.25, 0.40]
    with mp.Manager() as manager:
        out = manager.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), local_ms, out), nprocs=world, join=True)
        res = dict(out)
    import bench
    for rank in range(world):
        ms, value, skipped = res[rank]
        assert ms == pytest.approx(0.40)                           # max over ranks, on every rank
        assert value == pytest.approx(world * bench.FLOPS_STEP / 0.40e-3 / 1e12)
    assert res[1][2]                                               # rank 1 did no reference work


def test_single_rank_value():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_value(1, 1.0) == pytest.approx(bench.FLOPS_STEP / 1e-3 / 1e12)
