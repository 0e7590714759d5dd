"""The multi-rank bench path on CPU: two gloo ranks, each an independent
replica, aggregated as the slowest rank's time over the units of all ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dm = bench.make_dist_max(dist)
        dm("barrier")
        # rank r took (r + 1) * 10 ms for 4 steps of a 2-GFLOP replica
        ms, value = bench.aggregate(2e9, 10.0 * (rank + 1), 4, world, dm)
        out[rank] = (ms, value)
    finally:
        dist.destroy_process_group()


def test_aggregate_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    # both ranks see the slowest rank's time; the rate counts both replicas
    for r in range(world):
        ms, value = out[r]
        assert ms == pytest.approx(20.0)
        assert value == pytest.approx(2e9 * world / (20e-3 / 4) / 1e12)


def test_aggregate_single_process():
    ms, value = bench.aggregate(1e12, 5.0, 10, 1, None)
    assert ms == 5.0
    assert value == pytest.approx(1e12 / 0.5e-3 / 1e12)
