"""The multi-rank aggregation of bench.py (max time over ranks, whole-job
bytes) with world_size 2 over gloo on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    ms, nbytes = bench.reduce_ranks(torch, dist, ms=1.0 + rank, nbytes=100.0 * (rank + 1), device="cpu")
    out[rank] = (ms, nbytes)
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_ranks_world2_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        assert out[r] == (2.0, 300.0)


def test_reduce_ranks_single_process():
    import torch
    import bench
    assert bench.reduce_ranks(torch, None, 3.5, 7.0) == (3.5, 7.0)
