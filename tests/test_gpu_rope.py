"""GPU parity of the verify layer's neighbour: tree Q/K turned to position
P + depth (RoPE) and tree K/V written into the cache tail, against the
oracle (float64 rope and write_tree_kv).

The kernel computes the angles in fp64, rotates in fp32 and rounds to the
dtype: every rotated element is within half an ulp of the dtype (plus fp32
rounding) of the float64 value; V rows and every cache row outside the
tree slots are compared bit for bit.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import attention_ref, attn_close, raw_bits, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"
THETA = 1e6


def _tol(ref, dtype):
    rel = 2.0 ** -8 if dtype == torch.bfloat16 else 2.0 ** -22
    return rel * np.abs(ref) * 1.01 + 1e-5


def _inputs(w, rep=0):
    g = torch.Generator().manual_seed(1000 + 10 * w.cfg + rep)
    shape_q = (w.layers, w.N, w.n, w.Hq, w.D)
    shape_kv = (w.layers, w.N, w.n, w.Hkv, w.D)
    q = torch.randn(shape_q, generator=g).to(w.torch_dtype)
    k = torch.randn(shape_kv, generator=g).to(w.torch_dtype)
    v = torch.randn(shape_kv, generator=g).to(w.torch_dtype)
    return q, k, v


def _run(w, st, prefix, cache, q_in, k_in, v_in, theta=THETA):
    kd, vd = cache.k.to(CUDA), cache.v.to(CUDA)
    bt = None if cache.block_table is None else cache.block_table.to(CUDA)
    kv = dd.kv_desc_for(kd, w.N, w.Hq, bt)
    q_out = torch.full_like(q_in, 7.0).to(CUDA)
    dd.ddtree_tree_kv_write(k_in.to(CUDA), v_in.to(CUDA), torch.from_numpy(st["depth"]).to(CUDA),
                            torch.from_numpy(st["n_nodes"]).to(CUDA), prefix.to(CUDA), kv, kd, vd, w.B,
                            rope_theta=theta, q_in=q_in.to(CUDA), q_out=q_out, block_table=bt)
    torch.cuda.synchronize()
    return q_out.cpu(), kd.cpu(), vd.cpu()


@pytest.mark.parametrize("cfg,over", [(1, {}), (2, {}), (4, dict(N=5)), (3, dict(layers=3))])
def test_tree_kv_write_matches_oracle(cfg, over):
    w = datagen.workload(cfg, **over)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q_in, k_in, v_in = _inputs(w)
    q_out, kd, vd = _run(w, st, prefix, cache, q_in, k_in, v_in)
    assert dd.device_status() == 0
    P = prefix.numpy()
    table = None if cache.block_table is None else cache.block_table.numpy()
    # the oracle's cache after the write (float64), and the slots it wrote
    k_ref = cache.k.to(torch.float64).numpy().copy()
    v_ref = cache.v.to(torch.float64).numpy().copy()
    oracle.write_tree_kv(k_ref, v_ref, k_in.to(torch.float64).numpy(), v_in.to(torch.float64).numpy(),
                         st["depth"], P, st["n_nodes"], THETA, block_table=table)
    written = np.zeros(cache.k.shape[:3], bool)
    for r in range(w.N):
        slots = P[r] + np.arange(int(st["n_nodes"][r]))
        if table is None:
            written[:, r, slots] = True
        else:
            written[:, table[r, slots // 64], slots % 64] = True
    kg = kd.to(torch.float64).numpy()
    assert np.all(np.abs(kg[written] - k_ref[written]) <= _tol(k_ref[written], w.torch_dtype))
    assert np.array_equal(raw_bits(vd)[written], raw_bits(torch.from_numpy(v_ref).to(w.torch_dtype))[written])
    assert np.array_equal(raw_bits(kd)[~written], raw_bits(cache.k)[~written])
    assert np.array_equal(raw_bits(vd)[~written], raw_bits(cache.v)[~written])
    # Q of the live nodes rotated at the same positions; other rows untouched
    qo = q_out.to(torch.float64).numpy()
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        pos = oracle.tree_positions(st["depth"][r], int(P[r]), nn)
        for l in range(w.layers):
            ref = oracle.rope(q_in[l, r, :nn].to(torch.float64).numpy(), pos, THETA)
            assert np.all(np.abs(qo[l, r, :nn] - ref) <= _tol(ref, w.torch_dtype))
        assert np.all(qo[:, r, nn:] == 7.0)


def test_tree_kv_write_without_rotation_copies():
    w = datagen.workload(2)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q_in, k_in, v_in = _inputs(w, rep=1)
    q_out, kd, vd = _run(w, st, prefix, cache, q_in, k_in, v_in, theta=0.0)
    P = int(prefix[0])
    nn = int(st["n_nodes"][0])
    assert torch.equal(kd[:, 0, P:P + nn], k_in[:, 0, :nn])
    assert torch.equal(vd[:, 0, P:P + nn], v_in[:, 0, :nn])
    assert torch.equal(q_out[:, 0, :nn], q_in[:, 0, :nn])


def test_tree_kv_write_capacity_is_flagged():
    w = datagen.workload(1)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q_in, k_in, v_in = _inputs(w)
    big = torch.tensor([cache.s_max - 2], dtype=torch.int32)
    q_out, kd, vd = _run(w, st, big, cache, q_in, k_in, v_in)
    assert dd.device_status() & dd.STATUS_CAPACITY
    assert torch.equal(kd, cache.k)


@pytest.mark.parametrize("cfg", [2, 4])
def test_round_with_tree_kv_write(cfg):
    """The round rotates and writes the tree's Q/K/V after its build; the
    attention then sees them (oracle: write_tree_kv, rope, dense attention)."""
    w = datagen.workload(cfg, **({} if cfg == 2 else dict(N=4)))
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q_in, k_in, v_in = _inputs(w, rep=2)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    rb = dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B, kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=z.to(CUDA), root_token=torch.from_numpy(root).to(CUDA), q=torch.zeros_like(q_in).to(CUDA),
        k_cache=cache.k.to(CUDA), v_cache=cache.v.to(CUDA),
        block_table=None if cache.block_table is None else cache.block_table.to(CUDA),
        prefix_len=prefix.to(CUDA), target_logits=tgt.to(CUDA),
        tree_q_in=q_in.to(CUDA), tree_k_in=k_in.to(CUDA), tree_v_in=v_in.to(CUDA), rope_theta=THETA,
    ).allocate_outputs()
    assert dd.ddtree_round_launch_count(rb) >= 5
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    P = prefix.numpy()
    table = None if cache.block_table is None else cache.block_table.numpy()
    k_ref = cache.k.to(torch.float64).numpy().copy()
    v_ref = cache.v.to(torch.float64).numpy().copy()
    oracle.write_tree_kv(k_ref, v_ref, k_in.to(torch.float64).numpy(), v_in.to(torch.float64).numpy(),
                         st["depth"], P, st["n_nodes"], THETA, block_table=table)
    q_ref = np.zeros(q_in.shape)
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        pos = oracle.tree_positions(st["depth"][r], int(P[r]), nn)
        for l in range(w.layers):
            q_ref[l, r, :nn] = oracle.rope(q_in[l, r, :nn].to(torch.float64).numpy(), pos, THETA)
    ref_cache = datagen.KVCache(torch.from_numpy(k_ref), torch.from_numpy(v_ref), cache.block_table, cache.s_max)
    ref, _ = attention_ref(w, torch.from_numpy(q_ref), ref_cache, P, st["anc"], st["n_nodes"],
                           reqs=sorted({0, w.N - 1}), nodes=[0, 1, w.B // 2, w.B], heads=[0, 9, w.Hq - 1])
    for (l, r, i, h), v in ref.items():
        ok, ex = attn_close(rb.attn_out[l, r, i, h].to("cpu", torch.float64).numpy(), v)
        assert ok, (l, r, i, h, ex)
