"""GPU parity of the whole round (ddtree_round) against the oracle chain.

The round feeds its own top-K table to its build.  Its ids must equal the
oracle's and its log-probs lie within the stated tolerance of them (in
practice they are bit-identical: both are the fp64 log-softmax rounded once
to fp32).  The tree is then compared, bit for bit, with the oracle's tree
built from the round's own lp table ("DDTree Deep Dive" §2, Propositions 2
and 3: the tree is a function of that table), and with the oracle's own tree
when the tables agree.  Every downstream integer output and the compacted
cache are compared bit for bit, the attention output within tolerance.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import assert_topk, assert_tree, attention_ref, attn_close, np64, raw_bits, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def make_round(w, rep=0, gain_floor=None):
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w, rep)
    if gain_floor is not None:
        st = oracle.stack_trees(oracle.build_trees(ids, lp32, root, w.B, gain_floor=gain_floor))
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
        prefix_len=prefix.to(CUDA), target_logits=tgt.to(CUDA),
        gain_floor=None if gain_floor is None else torch.from_numpy(np.asarray(gain_floor, np.float32)).to(CUDA),
    ).allocate_outputs()
    host = dict(z=z, ids=ids, lp32=lp32, lse32=lse32, root=root, st=st, prefix=prefix.numpy(),
                cache=cache, q=q, tgt=tgt, gain_floor=gain_floor)
    return rb, host


def check_round(w, rb, h, layers=None, nodes=None, heads=None, reqs=None):
    assert dd.device_status() == 0
    assert_topk(rb.ids.reshape(-1, w.K), rb.lp.reshape(-1, w.K), rb.lse, h["ids"].reshape(-1, w.K),
                h["lp32"].reshape(-1, w.K), h["lse32"].reshape(-1))
    # the oracle's tree from the round's own (ids, lp) table: bit for bit
    g_ids = rb.ids.cpu().numpy()
    g_lp = rb.lp.cpu().numpy()
    own = oracle.stack_trees(oracle.build_trees(g_ids, g_lp, h["root"], w.B, gain_floor=h["gain_floor"]))
    assert_tree(rb.tree, own)
    st = h["st"]
    if np.array_equal(g_lp.view(np.uint32), h["lp32"].view(np.uint32)):
        assert_tree(rb.tree, st)
    else:
        st = own
    # attention of the tree nodes (sampled where asked)
    ref, _ = attention_ref(w, h["q"], h["cache"], h["prefix"], st["anc"], st["n_nodes"], layers=layers,
                           reqs=reqs, nodes=nodes, heads=heads)
    o = rb.attn_out
    for (l, r, i, hh), v in ref.items():
        got = o[l, r, i, hh].to("cpu", torch.float64).numpy()
        ok, ex = attn_close(got, v)
        assert ok, (l, r, i, hh, ex)
    # walk, and the compaction of every layer's K and V, bit for bit
    tg = h["tgt"]
    table = None if h["cache"].block_table is None else h["cache"].block_table.numpy()
    kh, vh = raw_bits(h["cache"].k), raw_bits(h["cache"].v)
    for r in range(w.N):
        a = oracle.accept(tg[r].to(torch.float64).numpy(), st["node_token"][r], st["parent"][r],
                          int(st["n_nodes"][r]), w.L, int(h["prefix"][r]))
        assert rb.acc.path[r].tolist() == a.path.tolist()
        assert int(rb.acc.accept_len[r]) == a.accept_len
        assert int(rb.acc.next_bonus[r]) == a.next_bonus
        assert int(rb.acc.new_prefix_len[r]) == a.new_prefix_len
        assert rb.acc.src_slot[r].tolist() == a.src_slot.tolist()
        assert rb.acc.dst_slot[r].tolist() == a.dst_slot.tolist()
        oracle.compact(kh, vh, r, a, block_table=table)
    assert np.array_equal(raw_bits(rb.k_cache), kh)
    assert np.array_equal(raw_bits(rb.v_cache), vh)


@pytest.mark.parametrize("cfg", [1, 2])
def test_round_configs(cfg):
    w = datagen.workload(cfg)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h)


def test_round_48_layers_b256_p8k():
    """b256_p8k_48l end to end: attention sampled over (layer, node, head),
    the walk's compaction of all 48 layers compared bit for bit (the separate
    walk + compaction launch)."""
    w = datagen.workload(3)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h, layers=[0, 23, 47], nodes=[0, 1, 100, 255, 256], heads=[0, 9, 31])


@pytest.mark.parametrize("sigma", [1.0, 8.0])
def test_round_p32k_b1024(sigma):
    """sweep_p32k at B = 1024: bushy (sigma 1) and chain-like (sigma 8) trees."""
    w = datagen.workload(5, B=1024, sigma=sigma)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h, nodes=[0, 1, 17, 512, 1023, 1024], heads=[0, 13, 31])


@pytest.mark.parametrize("floor_node", [None, 20])
def test_round_p32k_b64_split(floor_node):
    """sweep_p32k at B = 64 end to end: the two-M-tile attention split twelve
    ways inside the round, the splits holding prefix tiles only started while
    the tree is built; with a gain floor the tree stops short of the budget,
    so the attention tiles over more nodes than the tree has."""
    w = datagen.workload(5)
    assert dd.attn_plan(dd.kv_desc(1, 1, w.Hq, w.Hkv, w.D, s_max=32896), w.B) == ("two_mtile", 12)
    floor = None
    if floor_node is not None:
        z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
        floor = np.array([float(st["score"][0, floor_node])], np.float32)
    rb, h = make_round(w, gain_floor=floor)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    if floor_node is not None:
        assert int(rb.tree.n_nodes[0]) < w.n
    check_round(w, rb, h, nodes=[0, 1, 7, 15, 20] + ([] if floor_node else [40, 64]), heads=[0, 13, 31])


def test_round_batched_paged_sampled():
    w = datagen.workload(4)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h, nodes=[0, 3, 64], heads=[0, 31])


@pytest.mark.parametrize("cfg", [2, 4])
def test_round_adaptive_budget(cfg):
    """A round with per-request gain floors (adaptive budget): the build
    keeps the pops above each floor and every later stage works on that
    smaller tree."""
    w = datagen.workload(cfg)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    floor = np.array([float(st["score"][r, (7 * r + 20) % w.n]) for r in range(w.N)], np.float32)
    rb, h = make_round(w, gain_floor=floor)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    assert np.all(rb.tree.n_nodes.cpu().numpy() <= w.n)
    check_round(w, rb, h, nodes=None if cfg == 2 else [0, 3, 64], heads=None if cfg == 2 else [0, 31],
                reqs=None if cfg == 2 else [0, 5, 31])


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


def test_round_stage_events():
    """The round's stage events bracket its stages: five non-negative times
    whose sum is the round, with the attention the largest at 48 layers."""
    w = datagen.workload(3, layers=4)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    t = dd.ddtree_round_timed(rb)
    assert set(t) == set(dd.STAGES)
    assert all(v >= 0.0 for v in t.values())
    assert t["tree_kv_write"] < 0.05           # no tree K/V given: an empty stage
    assert t["attn"] == max(t.values())
