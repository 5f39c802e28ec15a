"""Pins of the CPU oracle to facts the pages and the mathematics fix.

None of these re-types an oracle formula: each compares the oracle with a
different route to the same answer (brute force, a library routine the
oracle does not use, a closed form, an invariant, or numbers printed on the
pages, stored under tests/golden/ with their citation).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from draft_tree_build_ddtree_b200 import datagen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _cfg1():
    w = datagen.workload(1)
    z = datagen.drafter_logits(w).to(torch.float64).numpy()
    ids, lp32, lse32, lp64 = oracle.topk(z, w.K)
    return w, z, ids, lp32, lse32, lp64


# ---------------------------------------------------------------- log-softmax

def test_log_softmax_normalises_and_matches_torch():
    g = torch.Generator().manual_seed(7)
    z = (torch.randn(6, 1000, generator=g, dtype=torch.float64) * 5).numpy()
    z[0, :10] = -np.inf
    lp, lse = oracle.log_softmax(z)
    assert np.all(np.abs(np.exp(lp).sum(-1) - 1.0) < 1e-12)
    ref = torch.log_softmax(torch.from_numpy(z), dim=-1).numpy()
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(lp))
    assert np.max(np.abs(lp[fin] - ref[fin])) < 1e-12
    ref_lse = torch.logsumexp(torch.from_numpy(z), dim=-1).numpy()
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def test_log_softmax_rejects_nan():
    z = np.zeros((2, 8))
    z[1, 3] = np.nan
    with pytest.raises(ValueError):
        oracle.log_softmax(z)


# ---------------------------------------------------------------- top-K

def _rank_by_counting(row, i):
    """Position of token i in (value desc, id asc): count who beats it."""
    v = row[i]
    return int(np.sum(row > v) + np.sum((row == v) & (np.arange(row.size) < i)))


@pytest.mark.parametrize("V,K", [(50, 7), (64, 64), (300, 33)])
def test_topk_ranks_by_counting_with_ties(V, K):
    g = torch.Generator().manual_seed(V * 31 + K)
    z = torch.randint(-4, 5, (5, V), generator=g).to(torch.float64).numpy()
    z[0, 3] = -0.0
    z[0, 4] = 0.0
    z[1, :5] = -np.inf
    ids, lp32, lse32, lp64 = oracle.topk(z, K)
    for r in range(z.shape[0]):
        ranks = [_rank_by_counting(z[r], int(i)) for i in ids[r]]
        assert ranks == list(range(K))
        assert lp32.dtype == np.float32
        assert np.all(lp32[r] == lp64[r, ids[r]].astype(np.float32))


def test_topk_signed_zero_and_neg_inf():
    z = np.array([[-0.0, 0.0, -np.inf, -1.0, -0.0]])
    ids, *_ = oracle.topk(z, 5)
    assert ids[0].tolist() == [0, 1, 4, 3, 2]


# ---------------------------------------------------------------- heap (Prop. 2, 3)

def test_prop2_heap_equals_bruteforce_config1():
    w, z, ids, lp32, *_ = _cfg1()
    t = oracle.build_tree(ids[0], lp32[0], 0, w.B)
    brute = oracle.bruteforce_top_prefixes(lp32[0], w.B)
    assert t.tuples[1:] == brute
    assert t.n_nodes == w.B + 1
    # prefix-closed, and parent indices point at the tuple's prefix
    index = {tup: i for i, tup in enumerate(t.tuples)}
    for i in range(1, t.n_nodes):
        tup = t.tuples[i]
        assert tup[:-1] in index
        assert index[tup[:-1]] == t.parent[i] < i
        assert t.depth[i] == len(tup)
        assert t.node_rank[i] == tup[-1]
        assert t.node_token[i] == ids[0, len(tup) - 1, tup[-1]]


@pytest.mark.parametrize("seed", range(6))
def test_prop2_heap_equals_bruteforce_with_exact_ties(seed):
    # A coarse table makes many prefixes tie exactly in fp32, so the
    # tuple tie-break decides the order.
    g = torch.Generator().manual_seed(100 + seed)
    L, K, B = 3, 4, 30
    lp = -torch.randint(0, 3, (L, K), generator=g).to(torch.float32).numpy()
    lp = -np.sort(-lp, axis=1)          # ranks sorted best-first like a top-K table
    ids = np.arange(L * K, dtype=np.int32).reshape(L, K)
    t = oracle.build_tree(ids, lp, 0, B)
    assert t.tuples[1:] == oracle.bruteforce_top_prefixes(lp, B)


def test_budget_larger_than_tree_space():
    lp = np.log(np.array([[0.5, 0.3], [0.6, 0.2]], dtype=np.float64)).astype(np.float32)
    ids = np.array([[5, 6], [7, 8]], dtype=np.int32)
    t = oracle.build_tree(ids, lp, 9, 100)
    assert t.n_nodes == 1 + 2 + 4
    assert np.all(t.parent[t.n_nodes:] == -1)
    assert np.all(t.anc[t.n_nodes:] == 0)


def test_prop1_expected_acceptance_config1():
    w, z, ids, lp32, lse32, lp64 = _cfg1()
    t = oracle.build_tree(ids[0], lp32[0], 0, w.B)
    lp64_topk = np.take_along_axis(lp64[0], ids[0].astype(np.int64), axis=-1)
    p_topk = np.exp(lp64_topk)
    lhs = oracle.expected_acceptance_enumerated(t, p_topk)
    rhs = oracle.surrogate_value(t.tuples, lp64_topk)
    assert abs(lhs - rhs) < 1e-9


def test_beam_and_chain_never_beat_heap():
    w, z, ids, lp32, lse32, lp64 = _cfg1()
    lp64_topk = np.take_along_axis(lp64[0], ids[0].astype(np.int64), axis=-1)
    heap = oracle.build_tree(ids[0], lp32[0], 0, w.B)
    v_heap = oracle.surrogate_value(heap.tuples, lp64_topk)
    for width in (1, 2, 3, 4):
        beam = oracle.beam_tree(lp32[0], width)
        assert len(beam) <= w.B
        assert oracle.surrogate_value(beam, lp64_topk) <= v_heap + 1e-15
    chain = oracle.chain_tree(w.L)
    assert oracle.surrogate_value(chain, lp64_topk) <= v_heap + 1e-15


def _brute_beam(lp32, width):
    """Beam search written from the definition over the full prefix list:
    at depth d, rank every length-d prefix whose parent is in the previous
    beam by reading R4 and keep the ``width`` best."""
    L, K = lp32.shape
    prev = {()}
    out = []
    for d in range(1, L + 1):
        cand = [u for u in itertools.product(range(K), repeat=d) if u[:-1] in prev]
        cand.sort(key=lambda u: (-float(oracle.prefix_score(lp32, u)), u))
        keep = cand[:width]
        out.extend(keep)
        prev = set(keep)
    return out


@pytest.mark.parametrize("width", [1, 2, 3, 5, 8])
def test_beam_tree_equals_definition_config1(width):
    w, z, ids, lp32, lse32, lp64 = _cfg1()
    beam = oracle.beam_tree(lp32[0], width)
    ref = _brute_beam(lp32[0], width)
    assert beam == ref
    # every depth keeps min(width, K * |previous beam|) prefixes
    K, L = w.K, w.L
    size, expect = 1, 0
    for _ in range(L):
        size = min(width, K * size)
        expect += size
    assert len(beam) == expect


def test_beam_tree_extremes():
    w, z, ids, lp32, lse32, lp64 = _cfg1()
    # width 1 is the single drafted line (argmax at every position)
    assert oracle.beam_tree(lp32[0], 1) == oracle.chain_tree(w.L)
    # a width no depth can fill keeps every prefix
    small = lp32[0][:3, :4]
    allp = [u for d in range(1, 4) for u in itertools.product(range(4), repeat=d)]
    assert sorted(oracle.beam_tree(small, 4 ** 3)) == sorted(allp)


def _prefix_closed_subsets(prefixes):
    """Every subset of ``prefixes`` whose members' parents are members."""
    idx = {u: i for i, u in enumerate(prefixes)}
    n = len(prefixes)
    for mask in range(1 << n):
        ok = True
        for u, i in idx.items():
            if (mask >> i) & 1 and len(u) > 1 and not (mask >> idx[u[:-1]]) & 1:
                ok = False
                break
        if ok:
            yield [u for u, i in idx.items() if (mask >> i) & 1]


@pytest.mark.parametrize("L,K,seed", [(2, 3, 0), (2, 3, 1), (3, 2, 2), (3, 2, 5)])
def test_adaptive_budget_equals_bruteforce_optimum(L, K, seed):
    """Reading R9 (Deep Dive §10, cost-aware budgets): the adaptive tree is
    the prefix-closed tree of at most B nodes that maximises
    sum_{u in T} q(u) - c * |T|, found here by trying every prefix-closed set."""
    g = torch.Generator().manual_seed(100 + seed)
    z = (torch.randn(L, 6, generator=g, dtype=torch.float64) * 1.5).numpy()
    ids, lp32, _, lp64 = oracle.topk(z, K)
    q = {}
    prefixes = [u for d in range(1, L + 1) for u in itertools.product(range(K), repeat=d)]
    lpk = np.take_along_axis(lp64, ids.astype(np.int64), axis=-1)
    for u in prefixes:
        q[u] = float(np.exp(sum(lpk[d, r] for d, r in enumerate(u))))
    vals = sorted(set(q.values()))
    # costs in the gaps between distinct gains (no gain within 1e-4 relative of c)
    costs = [0.5 * (a + b) for a, b in zip(vals, vals[1:]) if b - a > 1e-4 * b] + [vals[-1] * 1.5, vals[0] * 0.5]
    subsets = list(_prefix_closed_subsets(prefixes))
    for c in costs:
        for B in (1, 3, len(prefixes)):
            best = max((sum(q[u] for u in T) - c * len(T), sorted(T)) for T in subsets if len(T) <= B)
            t = oracle.build_tree(ids, lp32, 0, B, gain_floor=math.log(c))
            assert sorted(t.tuples[1:]) == best[1], (c, B)


def test_adaptive_budget_floor_edges():
    w, z, ids, lp32, lse32, lp64 = _cfg1()
    full = oracle.build_tree(ids[0], lp32[0], 0, w.B)
    # no floor and a floor below every score give the budgeted tree
    low = oracle.build_tree(ids[0], lp32[0], 0, w.B, gain_floor=-1e30)
    assert low.tuples == full.tuples
    # a floor at or above the best score keeps the root only; so does NaN
    for f in (0.0, float(full.score[1]), float("nan")):
        t = oracle.build_tree(ids[0], lp32[0], 0, w.B, gain_floor=f)
        assert t.n_nodes == 1 and t.tuples == [()]
    # a floor equal to a node's score drops that node and everything after it
    i = 7
    t = oracle.build_tree(ids[0], lp32[0], 0, w.B, gain_floor=float(full.score[i]))
    kept = [j for j in range(1, full.n_nodes) if full.score[j] > full.score[i]]
    assert t.n_nodes == 1 + len(kept)
    assert t.tuples == full.tuples[:t.n_nodes]


def test_lemma1_topk_min_b_v_suffices():
    g = torch.Generator().manual_seed(3)
    V, L = 9, 3
    z = (torch.randn(L, V, generator=g, dtype=torch.float64) * 2).numpy()
    for B in (2, 5, 8):
        K = min(B, V)
        ids_k, lp_k, *_ = oracle.topk(z, K)
        ids_v, lp_v, *_ = oracle.topk(z, V)
        tk = oracle.build_tree(ids_k, lp_k, 0, B)
        tv = oracle.build_tree(ids_v, lp_v, 0, B)
        assert tk.tuples == tv.tuples
        assert np.array_equal(tk.node_token, tv.node_token)


# ---------------------------------------------------------------- pages' examples

def test_worked_example_deep_dive():
    gold = _golden("worked_marginals_deep_dive.json")
    p = gold["position1"]
    toks = list(p)
    probs = np.array([p[t] for t in toks] + [1.0 - sum(p.values())])
    lp = np.log(probs)[None, :].astype(np.float32)          # L = 1
    ids = np.arange(probs.size, dtype=np.int32)[None, :]
    lp64 = np.log(probs)[None, :]
    greedy = oracle.build_tree(ids, lp, -1, 1)
    assert toks[greedy.node_token[1]] == gold["greedy_token"]
    three = oracle.build_tree(ids, lp, -1, 3)
    v1 = oracle.surrogate_value(greedy.tuples, lp64)
    v3 = oracle.surrogate_value(three.tuples, lp64)
    assert abs((v3 - v1) - gold["discarded_by_greedy"]) < 1e-6
    assert sorted(toks[i] for i in three.node_token[1:4]) == sorted(toks)


def test_example_marginals_llm_wiki_products():
    gold = _golden("example_marginals_llm_wiki.json")
    pos = gold["positions"]
    names = [list(d) for d in pos]
    probs = [np.array(list(d.values())) for d in pos]
    K = max(len(p) for p in probs)
    lp64 = np.full((2, K), -np.inf)
    for d in range(2):
        lp64[d, :len(probs[d])] = np.log(probs[d])
    # expected order from plain products, enumerated directly
    prods = []
    for d in (1, 2):
        for tup in itertools.product(*[range(len(probs[i])) for i in range(d)]):
            prods.append((-math.prod(probs[i][r] for i, r in enumerate(tup)), tup))
    prods.sort()
    for B in range(1, len(prods) + 1):
        t = oracle.build_tree(np.zeros((2, K), np.int32), lp64.astype(np.float32), 0, B)
        assert t.tuples[1:] == [tup for _, tup in prods[:B]]
    t = oracle.build_tree(np.zeros((2, K), np.int32), lp64.astype(np.float32), 0, 4)
    got = [names[len(u) - 1][u[-1]] for u in t.tuples[1:]]
    assert got == ["token_a", "token_b", "token_c", "token_x"]


def test_hand_tree_mask_block_diffusion_drafters():
    gold = _golden("hand_tree_block_diffusion_drafters.json")
    names = gold["nodes"]
    idx = {n: i for i, n in enumerate(names)}
    parent = np.array([-1] + [idx[gold["parent"][n]] for n in names[1:]], dtype=np.int32)
    anc = oracle.ancestor_mask(parent, len(names), len(names))
    row = int(anc[idx["D"], 0])
    seen = {n for n in names if (row >> idx[n]) & 1}
    assert seen == set(gold["attends"]["D"])
    assert not seen & set(gold["not_attends"]["D"])


def _walk_mask(parent, n_nodes, n):
    W = (n + 31) // 32
    m = np.zeros((n, W), np.uint32)
    for i in range(n_nodes):
        j = i
        while j >= 0:
            m[i, j // 32] |= np.uint32(1 << (j % 32))
            j = int(parent[j])
    return m


@pytest.mark.parametrize("seed", range(4))
def test_mask_equals_explicit_parent_walks(seed):
    g = torch.Generator().manual_seed(seed)
    L, V, B = 6, 40, 70
    z = (torch.randn(L, V, generator=g, dtype=torch.float64) * (1 + seed)).numpy()
    ids, lp32, *_ = oracle.topk(z, min(B, V))
    t = oracle.build_tree(ids, lp32, 1, B)
    assert np.array_equal(t.anc, _walk_mask(t.parent, t.n_nodes, B + 1))


# ---------------------------------------------------------------- attention

def _random_case(seed, N=2, layers=2, Hq=4, Hkv=2, D=16, L=4, V=30, B=9, paged=False):
    g = torch.Generator().manual_seed(seed)
    trees = []
    for r in range(N):
        z = (torch.randn(L, V, generator=g, dtype=torch.float64) * 2).numpy()
        ids, lp32, *_ = oracle.topk(z, min(B, V))
        trees.append(oracle.build_tree(ids, lp32, 0, B))
    st = oracle.stack_trees(trees)
    n = B + 1
    P = torch.randint(3, 12, (N,), generator=g).numpy().astype(np.int32)
    S = int(P.max()) + n
    q = torch.randn(layers, N, n, Hq, D, generator=g, dtype=torch.float64).numpy()
    k = torch.randn(layers, N, S, Hkv, D, generator=g, dtype=torch.float64).numpy()
    v = torch.randn(layers, N, S, Hkv, D, generator=g, dtype=torch.float64).numpy()
    return st, P, q, k, v


def _sdpa_reference(q, k, v, P, parent, n_nodes, scale, l, r):
    """torch SDPA (float64) with the boolean mask from explicit parent walks."""
    nn = int(n_nodes[r])
    Hq, Hkv = q.shape[3], k.shape[3]
    Pr = int(P[r])
    mask = torch.zeros(nn, Pr + nn, dtype=torch.bool)
    mask[:, :Pr] = True
    for i in range(nn):
        j = i
        while j >= 0:
            mask[i, Pr + j] = True
            j = int(parent[r, j])
    qq = torch.from_numpy(q[l, r, :nn]).permute(1, 0, 2)                 # [Hq, nn, D]
    kk = torch.from_numpy(k[l, r, :Pr + nn]).permute(1, 0, 2)
    vv = torch.from_numpy(v[l, r, :Pr + nn]).permute(1, 0, 2)
    kk = kk.repeat_interleave(Hq // Hkv, dim=0)
    vv = vv.repeat_interleave(Hq // Hkv, dim=0)
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=mask, scale=scale)
    return o.permute(1, 0, 2).numpy()                                     # [nn, Hq, D]


@pytest.mark.parametrize("seed", range(3))
def test_attention_equals_sdpa_with_mask(seed):
    st, P, q, k, v = _random_case(seed)
    scale = 1 / math.sqrt(q.shape[-1])
    out, _ = oracle.tree_attention(q, k, v, P, st["anc"], st["n_nodes"], scale)
    for l in range(q.shape[0]):
        for r in range(q.shape[1]):
            ref = _sdpa_reference(q, k, v, P, st["parent"], st["n_nodes"], scale, l, r)
            for i in range(int(st["n_nodes"][r])):
                for h in range(q.shape[3]):
                    assert np.max(np.abs(out[(l, r, i, h)] - ref[i, h])) < 1e-12


def test_attention_paged_equals_contiguous():
    st, P, q, k, v = _random_case(11)
    layers, N, S, Hkv, D = k.shape
    page = oracle.PAGE
    nb = (S + page - 1) // page
    perm = np.random.RandomState(0).permutation(N * nb)
    table = perm.reshape(N, nb).astype(np.int32)
    kp = np.zeros((layers, N * nb, page, Hkv, D))
    vp = np.zeros_like(kp)
    for r in range(N):
        for s in range(S):
            kp[:, table[r, s // page], s % page] = k[:, r, s]
            vp[:, table[r, s // page], s % page] = v[:, r, s]
    scale = 0.3
    a, _ = oracle.tree_attention(q, k, v, P, st["anc"], st["n_nodes"], scale)
    b, _ = oracle.tree_attention(q, kp, vp, P, st["anc"], st["n_nodes"], scale, block_table=table)
    for key in a:
        assert np.array_equal(a[key], b[key])


def test_attention_chain_is_causal():
    # chain tree: node i's ancestors are 0..i, so the tree part is causal
    n, P, H, D = 7, 5, 2, 8
    g = torch.Generator().manual_seed(5)
    parent = np.arange(-1, n - 1, dtype=np.int32)
    anc = oracle.ancestor_mask(parent, n, n)[None]
    q = torch.randn(1, 1, n, H, D, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, P + n, H, D, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, P + n, H, D, generator=g, dtype=torch.float64)
    out, _ = oracle.tree_attention(q.numpy(), k.numpy(), v.numpy(), np.array([P]), anc,
                                   np.array([n]), 0.5)
    # causal SDPA over the P+n sequence; the tree queries are its last n rows
    qs = torch.cat([torch.zeros(1, 1, P, H, D, dtype=torch.float64), q], dim=2)
    ref = torch.nn.functional.scaled_dot_product_attention(
        qs[0, 0].permute(1, 0, 2), k[0, 0].permute(1, 0, 2), v[0, 0].permute(1, 0, 2),
        is_causal=True, scale=0.5).permute(1, 0, 2)[P:]
    for i in range(n):
        for h in range(H):
            assert np.max(np.abs(out[(0, 0, i, h)] - ref[i, h].numpy())) < 1e-12


def test_attention_budget_zero_is_decode():
    P, H, D = 9, 3, 8
    g = torch.Generator().manual_seed(9)
    q = torch.randn(1, 1, 1, H, D, generator=g, dtype=torch.float64)
    k = torch.randn(1, 1, P + 1, H, D, generator=g, dtype=torch.float64)
    v = torch.randn(1, 1, P + 1, H, D, generator=g, dtype=torch.float64)
    anc = np.ones((1, 1, 1), np.uint32)
    out, _ = oracle.tree_attention(q.numpy(), k.numpy(), v.numpy(), np.array([P]), anc,
                                   np.array([1]), 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[0, 0].permute(1, 0, 2), k[0, 0].permute(1, 0, 2), v[0, 0].permute(1, 0, 2),
        scale=0.25).permute(1, 0, 2)
    for h in range(H):
        assert np.max(np.abs(out[(0, 0, 0, h)] - ref[0, h].numpy())) < 1e-12


def test_attention_uniform_keys_reveal_visible_set():
    # With all keys equal the softmax is uniform over the visible slots, so
    # one-hot values read the visible set back exactly.
    st, P, q, _, _ = _random_case(21, N=1, layers=1, Hq=2, Hkv=1, D=4, B=12)
    n = 13
    S = int(P[0]) + n
    k = np.zeros((1, 1, S, 1, 4))
    v = np.zeros((1, 1, S, 1, S))
    v[0, 0, np.arange(S), 0, np.arange(S)] = 1.0
    q2 = np.zeros((1, 1, n, 2, S))
    out, _ = oracle.tree_attention(q2, np.concatenate([k, np.zeros((1, 1, S, 1, S - 4))], -1),
                                   v, P, st["anc"], st["n_nodes"], 1.0)
    walk = _walk_mask(st["parent"][0], int(st["n_nodes"][0]), n)
    for i in range(int(st["n_nodes"][0])):
        vis = [j for j in range(n) if (int(walk[i, j // 32]) >> (j % 32)) & 1]
        expect = np.zeros(S)
        expect[:P[0]] = 1.0
        expect[P[0] + np.array(vis)] = 1.0
        expect /= expect.sum()
        assert np.max(np.abs(out[(0, 0, i, 0)] - expect)) < 1e-15


# ---------------------------------------------------------------- walk + compaction

def _deepest_consistent(t_arg, parent, node_token, n_nodes):
    """Brute force: the deepest node whose every edge matches the argmax above it."""
    best, best_depth = 0, 0
    for i in range(1, n_nodes):
        j, ok, d = i, True, 0
        while j > 0:
            p = int(parent[j])
            if node_token[j] != t_arg[p]:
                ok = False
                break
            j, d = p, d + 1
        if ok and d > best_depth:
            best, best_depth = i, d
    return best, best_depth


@pytest.mark.parametrize("seed", range(8))
def test_accept_equals_deepest_consistent_node(seed):
    g = torch.Generator().manual_seed(40 + seed)
    L, V, B = 5, 12, 25
    z = (torch.randn(L, V, generator=g, dtype=torch.float64) * 1.5).numpy()
    ids, lp32, *_ = oracle.topk(z, min(B, V))
    t = oracle.build_tree(ids, lp32, 3, B)
    n = B + 1
    target = torch.randn(n, V, generator=g, dtype=torch.float64).numpy()
    # plant matches along a random branch so long walks happen
    for i in range(1, t.n_nodes):
        if torch.rand(1, generator=g).item() < 0.5:
            target[t.parent[i], t.node_token[i]] = 10.0 + torch.rand(1, generator=g).item()
    acc = oracle.accept(target, t.node_token, t.parent, t.n_nodes, L, 100)
    tgt = np.argmax(target, axis=-1)
    last, depth = _deepest_consistent(tgt, t.parent, t.node_token, t.n_nodes)
    assert acc.accept_len == depth + 1
    assert acc.path[acc.accept_len - 1] == last
    assert acc.next_bonus == tgt[last]
    # the path is the ancestor chain of the last node
    chain = []
    j = last
    while j >= 0:
        chain.append(j)
        j = int(t.parent[j])
    assert acc.path[:acc.accept_len].tolist() == chain[::-1]
    assert acc.new_prefix_len == 100 + acc.accept_len
    assert acc.src_slot[:acc.accept_len].tolist() == [100 + j for j in chain[::-1]]


def test_accept_k1_chain_is_single_line():
    # K = 1, B = L: the tree is the single drafted line; acceptance is the
    # number of leading positions where the target argmax equals the draft.
    L, V = 6, 10
    g = torch.Generator().manual_seed(77)
    z = torch.randn(L, V, generator=g, dtype=torch.float64).numpy()
    ids, lp32, *_ = oracle.topk(z, 1)
    t = oracle.build_tree(ids, lp32, 4, L)
    assert list(t.parent[1:]) == list(range(L))
    draft = ids[:, 0]
    for n_match in range(L + 1):
        target = np.zeros((L + 1, V))
        for i in range(L + 1):
            target[i, (draft[i] + 1) % V if i < L else 0] = 1.0
        for i in range(n_match):
            target[i] = 0.0
            target[i, draft[i]] = 1.0
        acc = oracle.accept(target, t.node_token, t.parent, t.n_nodes, L, 0)
        lead = 0
        while lead < L and np.argmax(target[lead]) == draft[lead]:
            lead += 1
        assert acc.accept_len == lead + 1 == n_match + 1


def test_argmax_lowest_id_on_ties():
    x = np.array([[1.0, 3.0, 3.0, -1.0], [-0.0, 0.0, -1.0, 0.0]])
    assert oracle.argmax_rows(x).tolist() == [1, 0]


@pytest.mark.parametrize("paged", [False, True])
def test_compaction_equals_index_select(paged):
    g = torch.Generator().manual_seed(8)
    layers, N, S, Hkv, D = 2, 2, 40, 2, 4
    k = torch.randn(layers, N, S, Hkv, D, generator=g, dtype=torch.float64).numpy()
    v = torch.randn(layers, N, S, Hkv, D, generator=g, dtype=torch.float64).numpy()
    P = 7
    path = np.array([0, 2, 5, 9, 10, -1, -1], dtype=np.int32)
    acc = oracle.Acceptance(path, 5, 0, np.where(path >= 0, P + path, -1).astype(np.int32),
                            np.where(path >= 0, P + np.arange(7), -1).astype(np.int32),
                            P + 5, np.zeros(1, np.int32))
    src = torch.tensor([P + j for j in path[:5]])
    if not paged:
        k0, v0 = k.copy(), v.copy()
        oracle.compact(k, v, 1, acc)
        for c, c0 in ((k, k0), (v, v0)):
            expect = torch.index_select(torch.from_numpy(c0[:, 1]), 1, src).numpy()
            assert np.array_equal(c[:, 1, P:P + 5], expect)
            assert np.array_equal(c[:, 1, :P], c0[:, 1, :P])
            assert np.array_equal(c[:, 1, P + 5:], c0[:, 1, P + 5:])
            assert np.array_equal(c[:, 0], c0[:, 0])
    else:
        page = oracle.PAGE
        table = np.array([[1, 0], [3, 2]], dtype=np.int32)   # one page per request is enough here
        kp = torch.randn(layers, 4, page, Hkv, D, generator=g, dtype=torch.float64).numpy()
        vp = torch.randn(layers, 4, page, Hkv, D, generator=g, dtype=torch.float64).numpy()
        k0 = kp.copy()
        oracle.compact(kp, vp, 1, acc, block_table=table)
        logical = k0[:, table[1, 0]]                 # slots 0..63 of request 1
        expect = torch.index_select(torch.from_numpy(logical), 1, src).numpy()
        assert np.array_equal(kp[:, table[1, 0], P:P + 5], expect)


# ---------------------------------------------------------------- planted mistakes

def test_pins_catch_a_dropped_sibling_push():
    """A heap that never pushes siblings must fail the brute-force pin.

    Feeding the heap a one-column table is exactly a heap without sibling
    pushes: every popped entry then has only its child to push.
    """
    w, z, ids, lp32, *_ = _cfg1()
    t = oracle.build_tree(ids[0][:, :1], lp32[0][:, :1], 0, w.B)
    assert t.tuples[1:] != oracle.bruteforce_top_prefixes(lp32[0], w.B)


def test_pins_catch_a_wrong_scale_in_attention():
    st, P, q, k, v = _random_case(2)
    scale = 1 / math.sqrt(q.shape[-1])
    out, _ = oracle.tree_attention(q, k, v, P, st["anc"], st["n_nodes"], scale * 1.01)
    ref = _sdpa_reference(q, k, v, P, st["parent"], st["n_nodes"], scale, 0, 0)
    assert np.max(np.abs(out[(0, 0, 1, 0)] - ref[1, 0])) > 1e-6


# ---------------------------------------------------------------- temperature > 0 (reading R10)

@pytest.mark.parametrize("ctr,key", [((1, 0, 0, 0), (5, 7)), ((0, 6, 0, 0), (2 ** 64 - 1, 3)),
                                     ((17, 2, 9, 4), (123456789, 987654321))])
def test_philox4x64_matches_numpy_bit_generator(ctr, key):
    """The oracle's Philox4x64-10 against numpy's Philox bit generator (a
    library implementation of the same published generator), which first
    advances its 256-bit counter by one and then emits the four words."""
    c0, c1, c2, c3 = ctr
    start = (c0 - 1) % 2 ** 64, c1 - (1 if c0 == 0 else 0), c2, c3
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(start, dtype=np.uint64))
    raw = bg.random_raw(8)
    ours = oracle.philox4x64((np.array([c0, (c0 + 1) % 2 ** 64], dtype=np.uint64),
                              np.array([c1, c1 + (1 if c0 == 2 ** 64 - 1 else 0)], dtype=np.uint64), c2, c3), key)
    assert np.array_equal(ours.T.reshape(-1), raw)


def test_uniforms_are_open_unit_interval_and_distinct_per_counter():
    u = oracle.uniforms(1001, 3, 2, seed=11, offset=5)
    assert u.shape == (1001,) and np.all(u > 0.0) and np.all(u < 1.0)
    assert not np.array_equal(u, oracle.uniforms(1001, 4, 2, seed=11, offset=5))     # another node
    assert not np.array_equal(u, oracle.uniforms(1001, 3, 2, seed=11, offset=6))     # another round
    # a Kolmogorov-Smirnov distance consistent with uniform draws
    d = np.max(np.abs(np.sort(u) - (np.arange(1, 1002) - 0.5) / 1001))
    assert d < 1.63 / math.sqrt(1001) + 0.5 / 1001


def _chi2(counts, probs):
    n = counts.sum()
    e = probs * n
    return float(((counts - e) ** 2 / e).sum())


def test_sampling_follows_tempered_softmax():
    """Gumbel-max draws over many seeds follow softmax(z / T): chi-square
    with 4 degrees of freedom below its 1e-4 tail (23.5)."""
    z = np.array([1.0, 0.2, -0.5, 2.0, 0.0])
    T = 0.8
    p = np.exp(z / T - np.max(z / T))
    p /= p.sum()
    counts = np.zeros(5)
    for seed in range(20000):
        counts[oracle.sample_rows(z[None], T, seed, 0, 0)[0]] += 1
    assert _chi2(counts, p) < 23.5


def test_sampling_cold_limit_is_argmax():
    g = np.random.default_rng(4)
    x = np.round(g.normal(size=(6, 300)) * 100) / 100 + np.arange(300) * 1e-5   # distinct values
    assert np.array_equal(oracle.sample_rows(x, 1e-6, 9, 1, 0), oracle.argmax_rows(x))


def test_tree_walk_at_temperature_keeps_the_target_distribution():
    """Reading R10 on a two-level tree: the first committed token follows the
    root's tempered target distribution, and, when it is a tree child, the
    second one follows that child's (chi-square, 1e-4 tails)."""
    T = 1.3
    V = 4
    target = np.array([[0.5, 1.5, -1.0, 0.0],     # root
                       [1.0, -0.5, 0.3, 0.2],     # node 1 (token 1)
                       [0.0, 0.0, 2.0, -2.0],     # node 2 (token 0)
                       [0.4, 0.1, 0.1, 0.3]])     # node 3 (token 2, child of node 1)
    node_token = np.array([7, 1, 0, 2], np.int32)
    parent = np.array([-1, 0, 0, 1], np.int32)

    def pr(row):
        e = np.exp(target[row] / T - np.max(target[row] / T))
        return e / e.sum()
    first = np.zeros(V)
    second = {1: np.zeros(V), 2: np.zeros(V)}
    for seed in range(12000):
        t = oracle.sample_rows(target, T, seed, 0, 0)
        a = oracle.accept(target, node_token, parent, 4, 2, 0, tokens=t)
        toks = [int(node_token[n]) for n in a.path[1:a.accept_len]] + [a.next_bonus]
        first[toks[0]] += 1
        if a.accept_len >= 2:
            node = int(a.path[1])
            second[node][toks[1]] += 1
    assert _chi2(first, pr(0)) < 21.1            # 3 degrees of freedom
    assert _chi2(second[1], pr(1)) < 21.1
    assert _chi2(second[2], pr(2)) < 21.1


# ---------------------------------------------------------------- rotary positions (reading R11)

def test_rope_is_complex_rotation():
    """Half-split RoPE equals multiplying z_i = x_i + i x_{i+D/2} by
    exp(i pos theta^(-2i/D)) (numpy complex arithmetic)."""
    g = np.random.default_rng(2)
    x = g.normal(size=(5, 3, 16))
    pos = np.array([0, 1, 7, 300, 32768])
    theta = 1e6
    z = x[..., :8] + 1j * x[..., 8:]
    w = z * np.exp(1j * pos[:, None, None] * theta ** (-np.arange(8) * 2.0 / 16))
    ref = np.concatenate([w.real, w.imag], axis=-1)
    assert np.allclose(oracle.rope(x, pos, theta), ref, rtol=0, atol=1e-12)


def test_rope_properties():
    g = np.random.default_rng(3)
    q, k = g.normal(size=(1, 128)), g.normal(size=(1, 128))
    assert np.allclose(oracle.rope(q, [0], 1e6), q, atol=0)              # position 0: identity
    r = oracle.rope(q, [12345], 1e6)
    assert np.allclose(r[0, :64] ** 2 + r[0, 64:] ** 2, q[0, :64] ** 2 + q[0, 64:] ** 2, atol=1e-12)
    # the score depends on the relative position only
    for m, n, sft in ((5, 2, 100), (40000, 3, 777)):
        a = oracle.rope(q, [m], 1e6) @ oracle.rope(k, [n], 1e6).T
        b = oracle.rope(q, [m + sft], 1e6) @ oracle.rope(k, [n + sft], 1e6).T
        assert abs(float((a - b)[0, 0])) < 1e-9


def test_write_tree_kv_places_rotated_rows():
    g = np.random.default_rng(4)
    L_, N, n, H, D = 2, 2, 5, 1, 8
    k_in, v_in = g.normal(size=(L_, N, n, H, D)), g.normal(size=(L_, N, n, H, D))
    depth = np.array([[0, 1, 1, 2, -1], [0, 1, 2, 3, 4]])
    nn = np.array([4, 5])
    P = np.array([3, 0])
    kc, vc = np.zeros((L_, N, 12, H, D)), np.zeros((L_, N, 12, H, D))
    oracle.write_tree_kv(kc, vc, k_in, v_in, depth, P, nn, 1e4)
    for r in range(N):
        for i in range(nn[r]):
            assert np.allclose(kc[:, r, P[r] + i], oracle.rope(k_in[:, r, i], [P[r] + depth[r, i]] * L_, 1e4))
            assert np.array_equal(vc[:, r, P[r] + i], v_in[:, r, i])
    assert np.all(kc[:, 0, :3] == 0) and np.all(kc[:, 0, 7:] == 0)      # nothing outside the tree slots


# ---------------------------------------------------------------- LM-head argmax

def _hadamard(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def test_lm_head_argmax_orthogonal_rows():
    """Orthogonal (Hadamard) weight rows: hidden = a * row v gives logit a*d
    at v and 0 elsewhere, so the argmax is v (a > 0), and a row scaled by 2
    beats its own copy (lowest index only decides exact ties)."""
    d = 64
    W = _hadamard(d)
    hidden = np.stack([0.5 * W[7], 3.0 * W[0], 1.0 * W[63]])
    am, mx = oracle.lm_head_argmax(hidden, W)
    assert am.tolist() == [7, 0, 63]
    assert np.allclose(mx, [0.5 * d, 3.0 * d, 1.0 * d])
    W2 = np.concatenate([W, 2 * W[5:6], W[5:6]])          # rows 64 (2x row 5) and 65 (= row 5)
    am2, _ = oracle.lm_head_argmax(W[5:6], W2)
    assert am2.tolist() == [64]
    am3, _ = oracle.lm_head_argmax(W[9:10], np.concatenate([W, W[9:10]]))
    assert am3.tolist() == [9]                            # exact tie with row 64: the lower index
