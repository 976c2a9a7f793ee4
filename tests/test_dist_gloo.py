"""The multi-rank plumbing of bench.py (one replica per rank, max-over-ranks timing) on CPU with gloo."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        ms = bench.max_over_ranks(torch, dist, 10.0 * (rank + 1), device="cpu")
        out[rank] = (ms, bench.weak_scaling_rate(32768, w, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_weak_scaling_rate(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for rank in range(world):
        ms, rate = out[rank]
        assert ms == 10.0 * world                      # every rank sees the slowest rank's time
        assert rate == pytest.approx(32768 * world / (ms * 1e-3))


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(torch, None, 3.5) == 3.5
    assert bench.dist_env()[1] >= 1
