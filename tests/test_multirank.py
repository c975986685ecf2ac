"""The multi-rank path of bench.py on CPU: world_size 2 over gloo.

Decode sequences are independent, so N GPUs run N replicas with no data-path
collective; the only exchange is the max over ranks of the timings, checked
here with two gloo ranks on CPU."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, world, rank)
        local = [1.0 + rank, 10.0 - rank, 3.5]
        out[rank] = bench.reduce_max(local, "cpu")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    for r in range(world):
        assert out[r] == [2.0, 10.0, 3.5]


def test_reduce_max_single_process_is_identity():
    import bench
    assert bench.reduce_max([1.5, 2.0], "cpu") == [1.5, 2.0]
