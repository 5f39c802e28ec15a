"""Helpers shared by the GPU parity tests: oracle runs and comparisons.

Expected values come only from ``oracle``; inputs only from ``datagen``.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from draft_tree_build_ddtree_b200 import datagen

LP_TOL = 1e-5                 # |lp_gpu - lp_oracle| (absolute)
ATTN_ABS, ATTN_REL = 1e-2, 2e-2


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def oracle_topk(logits: torch.Tensor, K: int):
    """Oracle top-K of a CPU [..., V] tensor."""
    z = np64(logits)
    ids, lp32, lse32, _ = oracle.topk(z, K)
    return ids, lp32, lse32


def oracle_trees(ids: np.ndarray, lp32: np.ndarray, root: np.ndarray, B: int):
    trees = oracle.build_trees(ids, lp32, root, B)
    return trees, oracle.stack_trees(trees)


def assert_topk(ids_gpu, lp_gpu, lse_gpu, ids, lp32, lse32):
    gi = ids_gpu.cpu().numpy().reshape(ids.shape)
    assert np.array_equal(gi, ids), f"ids differ at {np.argwhere(gi != ids)[:5].tolist()}"
    gl = lp_gpu.cpu().numpy().reshape(lp32.shape)
    err = np.max(np.abs(gl.astype(np.float64) - lp32.astype(np.float64)))
    assert err <= LP_TOL, f"lp error {err}"
    if lse_gpu is not None:
        ge = lse_gpu.cpu().numpy().reshape(lse32.shape)
        fin = np.isfinite(lse32)
        assert np.max(np.abs(ge[fin].astype(np.float64) - lse32[fin])) <= LP_TOL * 4


def assert_tree(t_gpu, st: dict):
    """Bit-exact comparison of every tree array (score compared as bits)."""
    for name in ("node_token", "parent", "depth", "node_rank", "n_nodes"):
        g = getattr(t_gpu, name).cpu().numpy()
        e = st[name]
        assert np.array_equal(g, e), f"{name} differs at {np.argwhere(g != e)[:5].tolist()}"
    gs = t_gpu.score.cpu().numpy().view(np.uint32)
    es = st["score"].astype(np.float32).view(np.uint32)
    assert np.array_equal(gs, es), f"score bits differ at {np.argwhere(gs != es)[:5].tolist()}"
    ga = t_gpu.anc.cpu().numpy().view(np.uint32)
    assert np.array_equal(ga, st["anc"]), f"anc differs at {np.argwhere(ga != st['anc'])[:5].tolist()}"


def attn_close(got: np.ndarray, ref: np.ndarray):
    err = np.abs(got - ref)
    bound = ATTN_ABS + ATTN_REL * np.abs(ref)
    return bool(np.all(err <= bound)), float(np.max(err - bound))


def tree_inputs(w: datagen.Workload, rep: int = 0):
    """Drafter logits, the oracle's top-K table and trees for workload ``w``."""
    z = datagen.drafter_logits(w, rep)
    ids, lp32, lse32 = oracle_topk(z, w.K)
    root = datagen.root_tokens(w, rep).numpy()
    trees, st = oracle_trees(ids, lp32, root, w.B)
    return z, ids, lp32, lse32, root, trees, st


def order_margin(lp32: np.ndarray, B: int) -> float:
    """Smallest score gap among the first B+1 prefixes in the oracle's order.

    When it exceeds the accumulated log-prob tolerance, a GPU top-K table
    within tolerance of the oracle's yields the identical tree.  Two prefixes
    whose log-prob sequences are equal position by position tie
    exactly on both sides (same fp32 adds in the same order), so such pairs
    do not count.
    """
    t = oracle.build_tree(np.zeros(lp32.shape, np.int32), lp32, 0, B + 1)
    s = t.score[1:t.n_nodes].astype(np.float64)
    tups = t.tuples[1:t.n_nodes]
    margin = np.inf
    for a in range(len(tups) - 1):
        gap = s[a] - s[a + 1]
        if gap == 0.0:
            sa = [lp32[d, r] for d, r in enumerate(tups[a])]
            sb = [lp32[d, r] for d, r in enumerate(tups[a + 1])]
            if sa == sb:
                continue
        margin = min(margin, gap)
    return float(margin)


def raw_bits(t: torch.Tensor) -> np.ndarray:
    """The tensor's bytes as integers of its element size (exact comparisons
    and plain row copies without a float64 widening of large caches)."""
    t = t.detach().to("cpu").contiguous()
    if t.element_size() == 2:
        return t.view(torch.int16).numpy().copy()
    if t.element_size() == 4:
        return t.view(torch.int32).numpy().copy()
    return t.numpy().copy()


def attention_ref(w, q, cache, prefix, anc, n_nodes, layers=None, reqs=None, nodes=None, heads=None):
    """Oracle tree attention on sampled layers, widened to float64 one layer
    at a time (the 48-layer caches would not fit in float64 at once).
    Returns {(layer, req, node, head): out row} and the matching lse dict."""
    table = None if cache.block_table is None else cache.block_table.numpy()
    layers = range(q.shape[0]) if layers is None else layers
    out, lse = {}, {}
    for l in layers:
        o, s = oracle.tree_attention(np64(q[l:l + 1]), np64(cache.k[l:l + 1]), np64(cache.v[l:l + 1]), prefix,
                                     anc, n_nodes, datagen.default_scale(w), block_table=table, reqs=reqs,
                                     nodes=nodes, heads=heads)
        for (_, r, i, h), v in o.items():
            out[(l, r, i, h)] = v
            lse[(l, r, i, h)] = s[(0, r, i, h)]
    return out, lse
