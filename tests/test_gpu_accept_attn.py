"""GPU parity: verifier walk + KV compaction, and tree attention, against the oracle.

Trees come from the oracle; target logits and Q/K/V from the seeded
generators; the GPU stages receive exactly the oracle's inputs.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import attn_close, np64, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def _dev(x):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.to(CUDA)


def _target_for(w, z, st, rep=0, plant_path=None):
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]), rep)
    if plant_path is not None:
        # make the target agree with the draft along a deep branch of each request
        for r in range(w.N):
            j = plant_path[r]
            while j > 0:
                p = int(st["parent"][r, j])
                tgt[r, p, :] = -20.0
                tgt[r, p, int(st["node_token"][r, j])] = 20.0
                j = p
    return tgt


def _deepest(st, r):
    d = st["depth"][r, :st["n_nodes"][r]]
    return int(np.argmax(d))


def _run_accept(w, z, st, tgt, cache, prefix):
    kv = dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table) if cache is not None else None
    acc = dd.ddtree_accept(_dev(tgt), _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L,
                           _dev(prefix), cache.k if cache is not None else None,
                           cache.v if cache is not None else None, kv,
                           cache.block_table if cache is not None else None)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    return acc


def _check_accept(w, st, tgt, prefix, acc):
    tg = tgt.to(torch.float64).numpy()
    res = []
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        a = oracle.accept(tg[r], st["node_token"][r], st["parent"][r], nn, w.L, int(prefix[r]))
        assert acc.path[r].tolist() == a.path.tolist()
        assert int(acc.accept_len[r]) == a.accept_len
        assert int(acc.next_bonus[r]) == a.next_bonus
        assert acc.src_slot[r].tolist() == a.src_slot.tolist()
        assert acc.dst_slot[r].tolist() == a.dst_slot.tolist()
        assert int(acc.new_prefix_len[r]) == a.new_prefix_len
        ta = acc.target_argmax[r].cpu().numpy()
        assert np.array_equal(ta[:nn], a.target_argmax)
        assert np.all(ta[nn:] == -1)
        res.append(a)
    return res


def _cache_for(w, prefix, rep=0):
    c = datagen.kv_cache(w, torch.from_numpy(np.asarray(prefix)), rep)
    return c


def _to_dev_cache(c):
    return datagen.KVCache(c.k.to(CUDA), c.v.to(CUDA),
                           None if c.block_table is None else c.block_table.to(CUDA), c.s_max)


@pytest.mark.parametrize("cfg", [1, 2])
def test_accept_with_compaction(cfg):
    w = datagen.workload(cfg)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w).numpy()
    tgt = _target_for(w, z, st, plant_path=[_deepest(st, r) for r in range(w.N)])
    host = _cache_for(w, prefix)
    dev = _to_dev_cache(host)
    acc = _run_accept(w, z, st, tgt, dev, prefix)
    res = _check_accept(w, st, tgt, prefix, acc)
    kh, vh = np64(host.k), np64(host.v)
    for r, a in enumerate(res):
        assert a.accept_len > 1
        oracle.compact(kh, vh, r, a)
    assert np.array_equal(np64(dev.k.cpu()), kh)
    assert np.array_equal(np64(dev.v.cpu()), vh)


def test_accept_natural_targets_config2():
    w = datagen.workload(2)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w).numpy()
    tgt = _target_for(w, z, st)
    acc = _run_accept(w, z, st, tgt, None, prefix)
    _check_accept(w, st, tgt, prefix, acc)


def test_accept_paged_batched():
    w = datagen.workload(4)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w).numpy()
    plant = [_deepest(st, r) if r % 2 == 0 else 0 for r in range(w.N)]
    tgt = _target_for(w, z, st, plant_path=plant)
    host = _cache_for(w, prefix)
    dev = _to_dev_cache(host)
    acc = _run_accept(w, z, st, tgt, dev, prefix)
    res = _check_accept(w, st, tgt, prefix, acc)
    kh, vh = np64(host.k), np64(host.v)
    table = host.block_table.numpy()
    for r, a in enumerate(res):
        oracle.compact(kh, vh, r, a, block_table=table)
    assert np.array_equal(np64(dev.k.cpu()), kh)
    assert np.array_equal(np64(dev.v.cpu()), vh)


def test_accept_many_layers():
    w = datagen.workload(3, P=300)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w).numpy()
    tgt = _target_for(w, z, st, plant_path=[_deepest(st, 0)])
    host = _cache_for(w, prefix)
    dev = _to_dev_cache(host)
    acc = _run_accept(w, z, st, tgt, dev, prefix)
    (a,) = _check_accept(w, st, tgt, prefix, acc)
    kh, vh = np64(host.k), np64(host.v)
    oracle.compact(kh, vh, 0, a)
    assert np.array_equal(np64(dev.k.cpu()), kh)
    assert np.array_equal(np64(dev.v.cpu()), vh)


def test_accept_argmax_ties_pick_lowest_id():
    w = datagen.workload(2, V=4096)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    g = torch.Generator().manual_seed(3)
    tgt = torch.randint(-2, 3, (1, w.n, w.V), generator=g).to(torch.bfloat16)
    tgt[0, :, 0] = -0.0
    acc = _run_accept(w, z, st, tgt, None, np.array([10]))
    _check_accept(w, st, tgt, np.array([10]), acc)


def test_accept_capacity_violation_is_flagged_not_written():
    w = datagen.workload(1)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = np.array([w.P])
    host = _cache_for(w, prefix)
    dev = _to_dev_cache(host)
    before = dev.k.clone()
    tgt = _target_for(w, z, st, plant_path=[_deepest(st, 0)])
    kv = dd.kv_desc_for(dev.k, w.N, w.Hq)
    big = np.array([dev.s_max - 2])
    dd.ddtree_accept(_dev(tgt), _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L,
                     _dev(big), dev.k, dev.v, kv)
    assert dd.device_status() & dd.STATUS_CAPACITY
    assert torch.equal(before, dev.k)


# ------------------------------------------------------------------ attention

def _attn_case(w, rep=0):
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w, rep)
    prefix = datagen.prefix_lengths(w, rep)
    cache = datagen.kv_cache(w, prefix, rep)
    q = datagen.queries(w, rep)
    return st, prefix.numpy(), cache, q


def _gpu_attn(w, st, prefix, cache, q):
    dev = _to_dev_cache(cache)
    kv = dd.kv_desc_for(dev.k, w.N, w.Hq, dev.block_table)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=CUDA)
    out, _ = dd.ddtree_tree_attn(q.to(CUDA), dev.k, dev.v, kv, _dev(prefix), _dev(st["anc"]),
                                 _dev(st["n_nodes"]), w.B, dev.block_table, out_lse=lse)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    return out.cpu(), lse.cpu()


def _check_attn(w, st, prefix, cache, q, out, lse, **sample):
    table = None if cache.block_table is None else cache.block_table.numpy()
    ref, ref_lse = oracle.tree_attention(np64(q), np64(cache.k), np64(cache.v), prefix, st["anc"],
                                         st["n_nodes"], datagen.default_scale(w), block_table=table,
                                         **sample)
    o = np64(out)
    ls = lse.numpy()
    worst = -np.inf
    for (l, r, i, h), v in ref.items():
        ok, excess = attn_close(o[l, r, i, h], v)
        worst = max(worst, excess)
        assert ok, f"attention out of tolerance at layer {l} req {r} node {i} head {h}: {excess}"
        assert abs(ls[l, r, i, h] - ref_lse[(l, r, i, h)]) < 1e-3
    return worst


@pytest.mark.parametrize("cfg", [1, 2])
def test_attention_configs(cfg):
    w = datagen.workload(cfg)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse)


def test_attention_paged_batched_sampled():
    w = datagen.workload(4)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    # nodes 20 and 50 sit in M-tiles 1 and 3: the second M-tile of a two-M-tile CTA
    _check_attn(w, st, prefix, cache, q, out, lse, reqs=[0, 13, 31], nodes=[0, 1, 5, 20, 33, 50, 64],
                heads=[0, 7, 8, 31])


def test_attention_48_layers_sampled():
    w = datagen.workload(3)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse, layers=[0, 47], nodes=[0, 1, 128, 255, 256],
                heads=[0, 9, 31])


def test_attention_long_prefix_b1024_sampled():
    w = datagen.workload(5, B=1024, sigma=4.0)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse, nodes=[0, 1, 511, 1000, 1024], heads=[0, 31])


def _plan(w, cache):
    kv = dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table)
    return dd.attn_plan(kv, w.B, dd.BF16 if w.dtype == "bf16" else dd.F32)


def test_attention_two_mtile_every_row():
    """The two-M-tile kernel on 4 layers of the B = 256 tree over a
    1000-token prefix (a ragged last key tile; 17 M-tiles, so the last CTA's
    second M-tile has no rows): every node and head of two layers against
    the oracle."""
    w = datagen.workload(3, layers=4, P=1000)
    st, prefix, cache, q = _attn_case(w)
    assert _plan(w, cache) == ("two_mtile", 1)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse, layers=[0, 3])


def test_attention_two_mtile_split():
    """The two-M-tile kernel split twelve ways over a 32k prefix (B = 64),
    merged by the combine kernel: every node at four heads."""
    w = datagen.workload(5)
    st, prefix, cache, q = _attn_case(w)
    assert _plan(w, cache) == ("two_mtile", 12)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse, heads=[0, 7, 8, 31])


def test_attention_two_mtile_wait_timeout_reports_and_recovers():
    """The two-M-tile kernel's bounded waits: the producer withholds key
    tile 1, the MMA issuer's wait for it runs out after 200 us, every role
    leaves its loop, waits for its copies and products, frees the tensor
    memory and returns; the next call matches the oracle."""
    w = datagen.workload(3, layers=4, P=1000)
    st, prefix, cache, q = _attn_case(w)
    assert _plan(w, cache) == ("two_mtile", 1)
    lib = dd.lib()
    try:
        assert lib.ddtree_debug_attn_timeout(200_000, 1) == 0
        dev = _to_dev_cache(cache)
        kv = dd.kv_desc_for(dev.k, w.N, w.Hq, dev.block_table)
        dd.ddtree_tree_attn(q.to(CUDA), dev.k, dev.v, kv, _dev(prefix), _dev(st["anc"]), _dev(st["n_nodes"]), w.B)
        torch.cuda.synchronize()
        bits = dd.device_status()
        assert bits & dd.STATUS_TIMEOUT, bits
        assert not bits & dd.STATUS_SETUP
        assert dd.device_status() == 0
    finally:
        assert lib.ddtree_debug_attn_timeout(0, -1) == 0
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse, layers=[1], nodes=[0, 1, 100, 255, 256])


def test_attention_budget_zero_is_decode():
    w = datagen.workload(2, B=0, K=1)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse)


def test_accept_nan_rows_give_sentinel():
    """A target row of NaN only has no argmax: the kernel reports -1 (which
    matches no child, so the walk stops there) and flags NONFINITE; a row
    with some NaN entries takes the argmax of the others."""
    w = datagen.workload(2, V=4096)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    tgt = _target_for(w, z, st, plant_path=[_deepest(st, 0)])
    c = int(st["parent"][0, _deepest(st, 0)])     # a node on the planted path
    tgt[0, c, :] = float("nan")
    tgt[0, 0, 5:4000:7] = float("nan")            # the root row keeps its planted maximum
    acc = dd.ddtree_accept(_dev(tgt), _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L,
                           _dev(np.array([10])))
    torch.cuda.synchronize()
    assert dd.device_status() & dd.STATUS_NONFINITE
    ta = acc.target_argmax[0].cpu().numpy()
    assert ta[c] == -1
    clean = tgt[0, 0].clone()
    clean[torch.isnan(clean)] = -float("inf")
    assert ta[0] == int(oracle.argmax_rows(clean.to(torch.float64).numpy()[None])[0])
    path = [p for p in acc.path[0].tolist() if p >= 0]
    assert path[-1] == c and int(acc.next_bonus[0]) == -1
    assert int(acc.accept_len[0]) == len(path)


def test_attention_wait_timeout_reports_and_recovers():
    """The pipeline's bounded waits: with the producer withholding a key tile
    and a 200 us limit, a consumer wait runs out, the kernel returns and sets
    TIMEOUT (cleared by the status read), and the next call with the normal
    settings matches the oracle."""
    w = datagen.workload(2)
    st, prefix, cache, q = _attn_case(w)
    lib = dd.lib()
    try:
        assert lib.ddtree_debug_attn_timeout(200_000, 1) == 0
        dev = _to_dev_cache(cache)
        kv = dd.kv_desc_for(dev.k, w.N, w.Hq, dev.block_table)
        dd.ddtree_tree_attn(q.to(CUDA), dev.k, dev.v, kv, _dev(prefix), _dev(st["anc"]), _dev(st["n_nodes"]), w.B)
        torch.cuda.synchronize()
        bits = dd.device_status()
        assert bits & dd.STATUS_TIMEOUT, bits
        assert not bits & dd.STATUS_SETUP
        assert dd.device_status() == 0
    finally:
        assert lib.ddtree_debug_attn_timeout(0, -1) == 0
    assert lib.ddtree_debug_attn_timeout(0, -2) != 0
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    _check_attn(w, st, prefix, cache, q, out, lse)


@pytest.mark.parametrize("cfg,over", [(2, dict(D=64)), (4, dict(N=3, D=64)), (3, dict(layers=2, D=64)),
                                      (5, dict(B=256, K=256, D=64))])
def test_attention_bf16_d64_tensor_cores(cfg, over):
    """bf16 with head dim 64 runs on the tensor cores (two-M-tile kernel,
    split or not, contiguous or paged) and matches the oracle."""
    w = datagen.workload(cfg, **over)
    st, prefix, cache, q = _attn_case(w)
    out, lse = _gpu_attn(w, st, prefix, cache, q)
    sample = {} if cfg == 2 else dict(nodes=[0, 1, w.B // 2, w.B], heads=[0, 9, w.Hq - 1])
    if cfg == 4:
        sample["reqs"] = [0, w.N - 1]
    _check_attn(w, st, prefix, cache, q, out, lse, **sample)
