"""Host logic of the multi-rank benchmark on CPU: two gloo ranks report
different step times; every rank must see the slowest one, and the job
throughput counts both ranks' batches (weak scaling)."""
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


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 100.0 + 50.0 * rank          # rank 1 is the slow one
    m = bench.max_over_ranks(ms, dist, device="cpu")
    v = bench.job_throughput(world, 16 * 2048, 10, m)
    out[rank] = (m, v)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    assert out[0] == out[1]
    m, v = out[0]
    assert m == pytest.approx(150.0)
    assert v == pytest.approx(2 * 16 * 2048 * 10 / 0.150)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(12.5, None) == 12.5
    assert bench.job_throughput(1, 100, 4, 1000.0) == pytest.approx(400.0)
