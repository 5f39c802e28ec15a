"""Multi-rank plumbing on CPU (gloo, world size 2).

bench.py times each rank and reduces the time with a max over ranks; the
batched workload is sharded by request (request r on rank r mod world) and
each round's per-request outcome is all-gathered into request order
(draft_tree_build_ddtree_b200.serving).  These tests run that plumbing with
two CPU processes; the per-rank round is the CPU oracle here (test code),
the library's CUDA round on a GPU.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _env(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))


def _worker(rank, world, port, out):
    _env(rank, world, port)
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


def _oracle_accepts(w, reqs):
    """(accept_len, next_bonus, new_prefix_len) of the given requests, by the oracle."""
    import oracle
    from draft_tree_build_ddtree_b200 import datagen
    z = datagen.drafter_logits(w)
    ids, lp32, _, _ = oracle.topk(z.to(torch.float64).numpy(), w.K)
    root = datagen.root_tokens(w).numpy()
    st = oracle.stack_trees(oracle.build_trees(ids, lp32, root, w.B))
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    prefix = datagen.prefix_lengths(w).numpy()
    rows = []
    for r in reqs:
        a = oracle.accept(tgt[r].to(torch.float64).numpy(), st["node_token"][r], st["parent"][r],
                          int(st["n_nodes"][r]), w.L, int(prefix[r]))
        rows.append([a.accept_len, a.next_bonus, a.new_prefix_len])
    return torch.tensor(rows, dtype=torch.int32).reshape(len(reqs), 3)


def _shard_worker(rank, world, port, out):
    _env(rank, world, port)
    import bench
    from draft_tree_build_ddtree_b200 import datagen, serving
    bench.init_dist(world, backend="gloo")
    w = datagen.workload(1, N=7)
    mine = serving.shard_of(w.N, world, rank)
    local = _oracle_accepts(w, mine)
    out[rank] = serving.gather_by_request(local, w.N, world, rank).numpy()
    torch.distributed.destroy_process_group()


def test_sharded_accepts_equal_one_rank_run():
    """Seven requests over two ranks (4 + 3): every rank's gathered
    per-request outcome equals the one-rank run over all requests."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    from draft_tree_build_ddtree_b200 import datagen, serving
    w = datagen.workload(1, N=7)
    whole = _oracle_accepts(w, range(w.N)).numpy()
    assert np.array_equal(serving.gather_by_request(torch.from_numpy(whole), w.N, 1, 0).numpy(), whole)
    for rank in range(world):
        assert np.array_equal(out[rank], whole)


def test_shards_partition_the_batch():
    from draft_tree_build_ddtree_b200 import serving
    for n, world in ((32, 1), (32, 2), (32, 8), (7, 3), (2, 4)):
        parts = [serving.shard_of(n, world, r) for r in range(world)]
        assert sorted(x for p in parts for x in p) == list(range(n))
        assert all(all(x % world == r for x in p) for r, p in enumerate(parts))
    with pytest.raises(ValueError):
        serving.shard_of(4, 2, 2)


def test_bench_relaunches_under_torchrun():
    import bench
    cmd = bench.relaunch_cmd(["--gpus", "4", "--steps", "5"], 4, 29511)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=29511" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "5"]
    assert os.path.basename(cmd[-5]) == "bench.py"


def test_bench_rejects_world_size_mismatch(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.run_ours(bench.parse(["--gpus", "4"]))
