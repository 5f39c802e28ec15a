"""GPU parity of the round driven from host buffers (ddtree_round_host) and
of continuous rounds (serving.ServingLoop), against the oracle chain.

Continuous rounds: each round's accepted path is compacted into the cache,
the prefix grows by accept_len and the next bonus token becomes the next
root ("DDTree Deep Dive" §5 and §6); the oracle replays the same chain on the
host, round by round.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen, host_api, serving

from parity import assert_tree, attention_ref, attn_close, raw_bits, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def _round_buffers(w, z, root, q, cache, prefix, tgt):
    return dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B, kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=z.to(CUDA), root_token=torch.as_tensor(root).to(CUDA), q=q.to(CUDA),
        k_cache=cache.k.to(CUDA), v_cache=cache.v.to(CUDA),
        block_table=None if cache.block_table is None else cache.block_table.to(CUDA),
        prefix_len=prefix.to(CUDA), target_logits=tgt.to(CUDA)).allocate_outputs()


@pytest.mark.parametrize("cfg", [1, 2])
def test_round_from_host_buffers(cfg):
    """Device buffers start zeroed (the tree's K/V slots too); one
    ddtree_round_host call copies the host inputs in, runs the round and
    copies the results out, and they match the oracle."""
    w = datagen.workload(cfg)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q = datagen.queries(w)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    rb = _round_buffers(w, z, root, q, cache, prefix, tgt)
    real = rb
    host = host_api.make_host_round(real)           # pinned copies of the real inputs and tree K/V rows
    P = prefix.numpy()
    for t in (rb.drafter_logits, rb.q, rb.target_logits, rb.root_token, rb.prefix_len):
        t.zero_()
    for r in range(w.N):                            # the tree slots hold nothing yet
        rb.k_cache[:, r, P[r]:P[r] + w.n] = 0
        rb.v_cache[:, r, P[r]:P[r] + w.n] = 0
    host_api.round_from_host(rb, host, rb.args())
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    out = host.outputs
    for name in ("node_token", "parent", "n_nodes"):
        assert np.array_equal(out[name].numpy(), st[name]), name
    ref, _ = attention_ref(w, q, cache, P, st["anc"], st["n_nodes"], nodes=[0, 1, w.B // 2, w.B],
                           heads=[0, w.Hq - 1])
    for (l, r, i, h), v in ref.items():
        ok, ex = attn_close(out["attn_out"][l, r, i, h].to(torch.float64).numpy(), v)
        assert ok, (l, r, i, h, ex)
    for r in range(w.N):
        a = oracle.accept(tgt[r].to(torch.float64).numpy(), st["node_token"][r], st["parent"][r],
                          int(st["n_nodes"][r]), w.L, int(P[r]))
        assert out["path"][r].tolist() == a.path.tolist()
        assert int(out["accept_len"][r]) == a.accept_len
        assert int(out["next_bonus"][r]) == a.next_bonus
        assert int(out["new_prefix_len"][r]) == a.new_prefix_len
    es = 2 if w.dtype == "bf16" else 4
    expect_h2d = (z.numel() + q.numel() + tgt.numel()) * es + 2 * 4 * w.N + 2 * w.layers * w.N * w.n * w.Hkv * w.D * es
    assert host.h2d_bytes == expect_h2d


def test_round_from_host_concurrent_streams():
    """Two host-buffer rounds with disjoint device buffers, issued on two
    streams so that one round's copies overlap the other's kernels, give the
    same outputs, bit for bit, as the same rounds run one after the other."""
    w = datagen.workload(2)
    pairs = []
    for rep in (0, 1):
        z, ids, lp32, lse32, root, trees, st = tree_inputs(w, rep)
        prefix = datagen.prefix_lengths(w, rep)
        cache = datagen.kv_cache(w, prefix, rep)
        q = datagen.queries(w, rep)
        tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]), rep)
        rb = _round_buffers(w, z, root, q, cache, prefix, tgt)
        pairs.append((rb, host_api.make_host_round(rb)))
    ref = []
    for rb, host in pairs:
        host_api.round_from_host(rb, host, rb.args())
        torch.cuda.synchronize()
        ref.append({k: v.clone() for k, v in host.outputs.items()})
    for _, host in pairs:
        for v in host.outputs.values():
            v.zero_()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(4):
        for (rb, host), s in zip(pairs, streams):
            with torch.cuda.stream(s):
                host_api.round_from_host(rb, host, rb.args())
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    for (_, host), r in zip(pairs, ref):
        for k, v in r.items():
            assert torch.equal(host.outputs[k].view(torch.uint8), v.view(torch.uint8)), k


def test_round_from_host_rejects_paged_tree_rows():
    w = datagen.workload(4, N=2)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    rb = _round_buffers(w, z, root, datagen.queries(w), cache, prefix, tgt)
    host = host_api.make_host_round(rb)               # paged: no tree rows from the host
    assert host.inputs.get("tree_k") is None
    host_api.round_from_host(rb, host, rb.args())
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    keep = host.io.tree_k
    host.io.tree_k = host.io.drafter_logits           # any host pointer: the call must refuse it
    host.io.tree_v = host.io.drafter_logits
    with pytest.raises(dd.DDTreeError):
        host_api.round_from_host(rb, host, rb.args())
    host.io.tree_k = host.io.tree_v = keep


@pytest.mark.parametrize("cfg,over", [(4, dict(N=6)), (2, {})])
def test_serving_loop_continuous_rounds_match_oracle(cfg, over):
    w = datagen.workload(cfg, **over)
    rounds = 3
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix, extra_slots=rounds * (w.L + 1))
    q = datagen.queries(w)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    rb = _round_buffers(w, z, root, q, cache, prefix, tgt)
    loop = serving.ServingLoop(rb, serving.shard_of(w.N, 1, 0), w.N)
    kh, vh = raw_bits(cache.k), raw_bits(cache.v)
    table = None if cache.block_table is None else cache.block_table.numpy()
    P = prefix.numpy().astype(np.int64).copy()
    R = np.asarray(root).astype(np.int32).copy()
    tg = tgt.to(torch.float64).numpy()
    for k in range(rounds):
        stats = loop.step().cpu().numpy()
        torch.cuda.synchronize()
        assert dd.device_status() == 0
        stk = oracle.stack_trees(oracle.build_trees(ids, lp32, R, w.B))
        assert_tree(rb.tree, stk)
        now = datagen.KVCache(torch.from_numpy(kh.copy()).view(cache.k.dtype),
                              torch.from_numpy(vh.copy()).view(cache.v.dtype), cache.block_table, cache.s_max)
        ref, _ = attention_ref(w, q, now, P, stk["anc"], stk["n_nodes"], reqs=sorted({0, w.N - 1}),
                               nodes=[0, 1, w.B], heads=[0, w.Hq - 1])
        for (l, r, i, h), v in ref.items():
            ok, ex = attn_close(rb.attn_out[l, r, i, h].to("cpu", torch.float64).numpy(), v)
            assert ok, (k, l, r, i, h, ex)
        for r in range(w.N):
            a = oracle.accept(tg[r], stk["node_token"][r], stk["parent"][r], int(stk["n_nodes"][r]), w.L, int(P[r]))
            assert stats[r].tolist() == [a.accept_len, a.next_bonus, a.new_prefix_len], (k, r)
            oracle.compact(kh, vh, r, a, block_table=table)
            P[r] = a.new_prefix_len
            R[r] = a.next_bonus
        p_dev, r_dev = loop.committed()
        assert p_dev.cpu().numpy().tolist() == P.tolist()
        assert r_dev.cpu().numpy().tolist() == R.tolist()
    assert np.array_equal(raw_bits(rb.k_cache), kh)
    assert np.array_equal(raw_bits(rb.v_cache), vh)
