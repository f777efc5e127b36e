"""Host-side logic of the benchmark's multi-process path, run as two gloo
ranks on the CPU: the slowest rank sets the step time and the whole-job
value counts every rank's replica."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 100.0 - rank]  # rank 1 is slower on the first value
        got = bench.max_over_ranks(local, torch.device("cpu"))
        out[rank] = (got, bench.whole_job_tflops(1e12, world, got[0]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_value(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, value = out[r]
        assert got == [10.0 + world - 1, 100.0]
        assert abs(value - world * 1e12 / (got[0] * 1e-3) / 1e12) < 1e-9


def test_single_process_identity():
    import torch

    import bench
    assert bench.max_over_ranks([1.0, 2.0], torch.device("cpu")) == [1.0, 2.0]
    assert abs(bench.whole_job_tflops(2e12, 1, 1000.0) - 2.0) < 1e-12
