"""The N > 1 bench logic on CPU: two gloo ranks agree on the slowest rank's time and
report the whole-job throughput (weak scaling: each rank runs its own sequences)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    elapsed_ms = [40.0, 55.0][rank]               # per-rank device time of K steps
    mx = bench.max_over_ranks(elapsed_ms, world, device="cpu")
    value = bench.job_throughput(4096, 10, world, mx)
    out[rank] = (mx, value)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_and_throughput():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn")
    assert out[0] == out[1]
    mx, value = out[0]
    assert mx == 55.0
    assert value == pytest.approx(2 * 4096 * 10 / 0.055)


def test_single_rank_throughput_formula():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.job_throughput(4096, 1000, 1, 382.0) == pytest.approx(4096 * 1000 / 0.382)
