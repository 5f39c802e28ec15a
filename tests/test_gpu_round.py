"""GPU parity of the whole round (ddtree_round) against the oracle chain.

The round feeds its own top-K table to its build.  Its log-probs are the
fp64 log-softmax rounded once to fp32, like the oracle's, so the table is
bit-identical in practice and every tree array is then compared bit for
bit; every downstream integer output and the compacted cache are compared
bit for bit, the attention output within tolerance.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import assert_topk, attn_close, np64, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def make_round(w, rep=0):
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w, rep)
    prefix = datagen.prefix_lengths(w, rep)
    cache = datagen.kv_cache(w, prefix, rep)
    q = datagen.queries(w, rep)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]), rep)
    rb = dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B,
        kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=z.to(CUDA), root_token=torch.from_numpy(root).to(CUDA), q=q.to(CUDA),
        k_cache=cache.k.to(CUDA), v_cache=cache.v.to(CUDA),
        block_table=None if cache.block_table is None else cache.block_table.to(CUDA),
        prefix_len=prefix.to(CUDA), target_logits=tgt.to(CUDA)).allocate_outputs()
    host = dict(z=z, ids=ids, lp32=lp32, lse32=lse32, root=root, st=st, prefix=prefix.numpy(),
                cache=cache, q=q, tgt=tgt)
    return rb, host


def _valid_tree(parent, anc, n_nodes):
    for i in range(1, n_nodes):
        assert 0 <= parent[i] < i
    walk = oracle.ancestor_mask(parent, n_nodes, parent.shape[0])
    assert np.array_equal(anc.view(np.uint32), walk)


def check_round(w, rb, h, layers=None, nodes=None, heads=None):
    assert dd.device_status() == 0
    assert_topk(rb.ids.reshape(-1, w.K), rb.lp.reshape(-1, w.K), rb.lse, h["ids"].reshape(-1, w.K),
                h["lp32"].reshape(-1, w.K), h["lse32"].reshape(-1))
    st = h["st"]
    # The tree is a deterministic function of the (ids, lp) table, and the
    # build stage alone is bit-exact on identical tables; so when the round's
    # lp table is bit-identical to the oracle's, every tree array must be too.
    lp_same = np.array_equal(rb.lp.cpu().numpy().reshape(h["lp32"].shape).view(np.uint32),
                             h["lp32"].view(np.uint32))
    t = rb.tree
    if lp_same:
        for name in ("node_token", "parent", "depth", "node_rank", "n_nodes"):
            assert np.array_equal(getattr(t, name).cpu().numpy(), st[name]), name
        assert np.array_equal(t.anc.cpu().numpy().view(np.uint32), st["anc"])
        assert np.array_equal(t.score.cpu().numpy().view(np.uint32), st["score"].view(np.uint32))
    else:
        for r in range(w.N):
            _valid_tree(t.parent[r].cpu().numpy(), t.anc[r].cpu().numpy(), int(t.n_nodes[r]))
        pytest.skip("an lp value differs from the oracle's in its last bit: tree validity checked only")
    # attention of the tree nodes
    table = None if h["cache"].block_table is None else h["cache"].block_table.numpy()
    ref, _ = oracle.tree_attention(np64(h["q"]), np64(h["cache"].k), np64(h["cache"].v), h["prefix"],
                                   st["anc"], st["n_nodes"], datagen.default_scale(w), block_table=table,
                                   layers=layers, nodes=nodes, heads=heads)
    o = np64(rb.attn_out.cpu())
    for (l, r, i, hh), v in ref.items():
        ok, ex = attn_close(o[l, r, i, hh], v)
        assert ok, (l, r, i, hh, ex)
    # walk and compaction
    tg = h["tgt"].to(torch.float64).numpy()
    kh, vh = np64(h["cache"].k), np64(h["cache"].v)
    for r in range(w.N):
        a = oracle.accept(tg[r], st["node_token"][r], st["parent"][r], int(st["n_nodes"][r]), w.L,
                          int(h["prefix"][r]))
        assert rb.acc.path[r].tolist() == a.path.tolist()
        assert int(rb.acc.accept_len[r]) == a.accept_len
        assert int(rb.acc.next_bonus[r]) == a.next_bonus
        assert int(rb.acc.new_prefix_len[r]) == a.new_prefix_len
        oracle.compact(kh, vh, r, a, block_table=table)
    assert np.array_equal(np64(rb.k_cache.cpu()), kh)
    assert np.array_equal(np64(rb.v_cache.cpu()), vh)


@pytest.mark.parametrize("cfg", [1, 2])
def test_round_configs(cfg):
    w = datagen.workload(cfg)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h)


def test_round_batched_paged_sampled():
    w = datagen.workload(4)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h, nodes=[0, 3, 64], heads=[0, 31])


@pytest.mark.parametrize("cfg,over", [
    (1, dict(N=3)),                      # 12 rows of 512 logits: one chunk per row
    (2, dict(N=2, V=32768)),             # 32 rows, 4 chunks each: 128 CTAs
    (2, dict(N=2, V=32768, B=0)),        # root-only trees
])
def test_round_multi_request(cfg, over):
    """Several requests in one round, each with exactly its own tree, and a
    second round on the same workspace (tickets back at zero) repeats it."""
    w = datagen.workload(cfg, **over)
    rb, h = make_round(w)
    args = rb.args()
    k0, v0 = rb.k_cache.clone(), rb.v_cache.clone()
    dd.ddtree_round(rb, args)
    torch.cuda.synchronize()
    check_round(w, rb, h, nodes=sorted({0, min(1, w.B), w.B // 2, w.B}), heads=[0, w.Hq - 1])
    # the per-request tickets are back at zero: a second round builds the same trees
    first = [x.clone() for x in (rb.tree.parent, rb.tree.anc, rb.tree.n_nodes, rb.acc.path)]
    rb.k_cache.copy_(k0)
    rb.v_cache.copy_(v0)
    dd.ddtree_round(rb, args)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    for a, b in zip(first, (rb.tree.parent, rb.tree.anc, rb.tree.n_nodes, rb.acc.path)):
        assert torch.equal(a, b)


def test_round_launch_count():
    """The launch plan the round reports: top-K, build, attention (+ the
    combine when b64_p2k splits its key range), argmax (+ a separate walk
    and compaction launch above two cache layers)."""
    rb2, _ = make_round(datagen.workload(2))
    assert dd.ddtree_round_launch_count(rb2) == 5
    rb1, _ = make_round(datagen.workload(1))
    assert dd.ddtree_round_launch_count(rb1) == 4
    rb1l, _ = make_round(datagen.workload(1, layers=3))
    assert dd.ddtree_round_launch_count(rb1l) == 5


def test_round_repeats_are_identical():
    w = datagen.workload(2)
    rb, h = make_round(w)
    args = rb.args()
    k0, v0 = rb.k_cache.clone(), rb.v_cache.clone()
    dd.ddtree_round(rb, args)
    first = [x.clone() for x in (rb.ids, rb.lp, rb.tree.anc, rb.attn_out, rb.acc.path)]
    rb.k_cache.copy_(k0)
    rb.v_cache.copy_(v0)
    dd.ddtree_round(rb, args)
    torch.cuda.synchronize()
    for a, b in zip(first, (rb.ids, rb.lp, rb.tree.anc, rb.attn_out, rb.acc.path)):
        assert torch.equal(a, b)
