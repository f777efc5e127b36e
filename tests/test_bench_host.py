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


def test_peak_choice_follows_the_clock():
    import bench
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    at_max = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0}
    capped = {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0}
    assert bench.choose_peak(peaks, at_max, 0.6) == (1600.0, "burst")
    assert bench.choose_peak(peaks, capped, 0.6) == (1400.0, "sustained")
    assert bench.choose_peak(peaks, at_max, 5000.0) == (1400.0, "sustained")
    assert bench.choose_peak(peaks, {"sm_mhz": None, "sm_max_mhz": None}, 0.6)[1] == "sustained"


def test_visible_pair_counts():
    """FLOP counts of the masked variants: closed forms for the causal and
    local-window masks, brute force for a tile mask."""
    import numpy as np

    import bench
    N = 300
    assert bench.visible_pairs(N) == N * N
    assert bench.visible_pairs(N, -1, 0) == N * (N + 1) // 2
    w = 37  # query i sees keys max(0, i - w) .. i
    assert bench.visible_pairs(N, w, 0) == sum(min(i, w) + 1 for i in range(N))
    T = (N + 127) // 128
    tm = np.array([[1, 0, 1], [0, 1, 0], [1, 1, 1]], dtype=bool)[:T, :T]
    brute = sum(1 for i in range(N) for j in range(N) if j <= i and tm[i // 128, j // 128])
    assert bench.visible_pairs(N, -1, 0, tm) == brute
    assert bench.visible_pairs(N, -1, -1, np.ones((T, T), bool)) == N * N
