"""GPU parity of verification at temperature > 0 (ddtree_accept_ex and the
round's sampling option) against the oracle's draws (oracle.sample_rows:
Philox4x64-10 uniforms, Gumbel-max, fp64 score rounded once to fp32).

Both sides form the perturbed score in fp64 and take the argmax in fp32; the
only operation that is not correctly rounded is the fp64 log (CUDA's and the
host's may differ in the last bit), so a draw may differ only where the two
best perturbed scores lie within a few fp32 ulps of each other.  Such
mismatches are accepted after that margin is checked; everything else is
compared bit for bit.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import raw_bits, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def _dev(x):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.to(CUDA)


def _scores32(row, T, seed, offset, req, node):
    u = oracle.uniforms(row.shape[0], node, req, seed, offset)
    return (np.asarray(row, np.float64) * (1.0 / T) - np.log(-np.log(u))).astype(np.float32)


def _check_draws(got, tgt, nn, T, seed, offset, req):
    """got: drawn tokens of the live nodes; returns the oracle's draws (with
    near-tie mismatches replaced by the GPU's choice after the margin check)."""
    x = tgt[:nn].to(torch.float64).numpy()
    ref = oracle.sample_rows(x, T, seed, offset, req)
    out = ref.copy()
    for i in np.nonzero(got[:nn] != ref)[0]:
        s = _scores32(x[i], T, seed, offset, req, int(i))
        a, b = float(s[ref[i]]), float(s[got[i]])
        assert abs(a - b) <= 4 * np.spacing(np.float32(abs(a))), (i, ref[i], got[i], a, b)
        out[i] = got[i]
    return out


@pytest.mark.parametrize("cfg,T,seed", [(1, 0.7, 1), (1, 2.5, 2), (2, 1.0, 3), (2, 0.6, 4)])
def test_accept_sampled_matches_oracle(cfg, T, seed):
    w = datagen.workload(cfg)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w).numpy()
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    cache = datagen.kv_cache(w, torch.from_numpy(prefix))
    kd, vd = cache.k.to(CUDA), cache.v.to(CUDA)
    kv = dd.kv_desc_for(kd, w.N, w.Hq)
    offset = 17
    acc = dd.ddtree_accept(_dev(tgt), _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L,
                           _dev(prefix), kd, vd, kv, temperature=T, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    kh, vh = raw_bits(cache.k), raw_bits(cache.v)
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        got = acc.target_argmax[r].cpu().numpy()
        draws = _check_draws(got, tgt[r], nn, T, seed, offset, r)
        assert np.all(got[nn:] == -1)
        a = oracle.accept(tgt[r].to(torch.float64).numpy(), st["node_token"][r], st["parent"][r], nn, w.L,
                          int(prefix[r]), tokens=draws)
        assert acc.path[r].tolist() == a.path.tolist()
        assert int(acc.accept_len[r]) == a.accept_len
        assert int(acc.next_bonus[r]) == a.next_bonus
        assert int(acc.new_prefix_len[r]) == a.new_prefix_len
        oracle.compact(kh, vh, r, a)
    assert np.array_equal(raw_bits(kd), kh)
    assert np.array_equal(raw_bits(vd), vh)


def test_sampling_reproducible_and_keyed():
    """The same (seed, offset) draws the same tokens; another offset (the
    next round) draws others; temperature <= 0 is the greedy argmax."""
    w = datagen.workload(2)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    tgt = _dev(datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"])))
    args = (tgt, _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L, _dev(np.array([5])))
    a1 = dd.ddtree_accept(*args, temperature=1.0, seed=9, offset=1).target_argmax.clone()
    a2 = dd.ddtree_accept(*args, temperature=1.0, seed=9, offset=1).target_argmax.clone()
    a3 = dd.ddtree_accept(*args, temperature=1.0, seed=9, offset=2).target_argmax.clone()
    g0 = dd.ddtree_accept(*args, temperature=0.0, seed=9, offset=1).target_argmax.clone()
    g1 = dd.ddtree_accept(*args).target_argmax.clone()
    torch.cuda.synchronize()
    assert torch.equal(a1, a2)
    assert not torch.equal(a1, a3)
    assert torch.equal(g0, g1)
    with pytest.raises(dd.DDTreeError):
        dd.ddtree_accept(*args, temperature=float("nan"))


def test_sampling_cold_limit_is_greedy():
    """fp32 targets with distinct values: a tiny temperature draws the argmax."""
    w = datagen.workload(1)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    args = (_dev(tgt), _dev(st["node_token"]), _dev(st["parent"]), _dev(st["n_nodes"]), w.L, _dev(np.array([3])))
    cold = dd.ddtree_accept(*args, temperature=1e-7, seed=1).target_argmax.clone()
    greedy = dd.ddtree_accept(*args).target_argmax.clone()
    torch.cuda.synchronize()
    assert torch.equal(cold, greedy)


def test_round_with_sampling_matches_oracle_chain():
    w = datagen.workload(4, N=4)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q = datagen.queries(w)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    T, seed, offset = 0.8, 1234, 3
    rb = dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B, kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=z.to(CUDA), root_token=torch.from_numpy(root).to(CUDA), q=q.to(CUDA),
        k_cache=cache.k.to(CUDA), v_cache=cache.v.to(CUDA), block_table=cache.block_table.to(CUDA),
        prefix_len=prefix.to(CUDA), target_logits=tgt.to(CUDA), sampling=dd.Sampling(T, seed, offset),
    ).allocate_outputs()
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    kh, vh = raw_bits(cache.k), raw_bits(cache.v)
    table = cache.block_table.numpy()
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        draws = _check_draws(rb.acc.target_argmax[r].cpu().numpy(), tgt[r], nn, T, seed, offset, r)
        a = oracle.accept(tgt[r].to(torch.float64).numpy(), st["node_token"][r], st["parent"][r], nn, w.L,
                          int(prefix[r]), tokens=draws)
        assert rb.acc.path[r].tolist() == a.path.tolist()
        assert int(rb.acc.next_bonus[r]) == a.next_bonus
        oracle.compact(kh, vh, r, a, block_table=table)
    assert np.array_equal(raw_bits(rb.k_cache), kh)
    assert np.array_equal(raw_bits(rb.v_cache), vh)
