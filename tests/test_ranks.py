"""The bench's multi-GPU bookkeeping on CPU: two gloo ranks, each with its
own time, must both see the slowest rank's time, and throughput must count
every rank's units (weak scaling, replicas only)."""

import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [0.5, 2.0][rank]
        out[rank] = bench.max_over_ranks(mine, dist, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 2.0, 1: 2.0}


def test_single_rank_and_aggregate():
    assert bench.max_over_ranks(1.25, None, "cpu") == 1.25
    a = bench.aggregate(weights_per_rank_step=1000, steps=10, world=4, t_slowest=2.0)
    assert a["value"] == pytest.approx(1000 * 10 * 4 / 2.0)
    assert a["ms_per_step"] == pytest.approx(200.0)
