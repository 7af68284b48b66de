"""The benchmark's multi-rank path on CPU: two gloo ranks take the max of their
timed regions and report whole-job throughput (replicas, weak scaling)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [120.0, 150.0][rank]
        ms_max = bench.max_over_ranks(torch, dist, local_ms, torch.device("cpu"), world)
        out[rank] = (ms_max, bench.job_tokens_per_s(world, 64, 100, ms_max))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        ms_max, value = res[rank]
        assert ms_max == 150.0
        assert value == pytest.approx(2 * 64 * 100 / 0.150)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(torch, None, 7.5, torch.device("cpu"), 1) == 7.5
    assert bench.job_tokens_per_s(1, 64, 10, 10.0) == pytest.approx(64 * 10 / 0.010)
