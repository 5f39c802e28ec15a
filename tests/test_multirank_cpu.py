"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

Each rank runs independent rounds (replicas); the only collectives are the
max-over-ranks reduction of the timed region and barriers.  These tests run
that plumbing with two CPU processes.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    bench.init_dist(world, backend="gloo")
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    bench.barrier()
    # rank 1 is the slow one: every rank must see its time
    t = bench.max_over_ranks(10.0 + 5.0 * rank)
    rate = bench.aggregate_rate(100, world, t / 1e3)
    out[rank] = (t, rate)
    torch.distributed.destroy_process_group()


def test_max_over_ranks_and_rate_two_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for rank in range(world):
        t, rate = out[rank]
        assert t == 15.0
        assert rate == pytest.approx(100 * world / 0.015)


def test_single_process_needs_no_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_rate(10, 1, 2.0) == 5.0
