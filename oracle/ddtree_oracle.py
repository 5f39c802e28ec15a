"""CPU oracle for one DDTree draft-and-verify round (test infrastructure).

This module is the checker, not the product.  Only the test suite, the
package's smoke check and the benchmark's CPU-baseline arm may import it; the
library never calls it and has no CPU fallback.  It shares no code with the
CUDA path: plain numpy, float64 unless the method fixes another precision,
no blocking, no fusion, loops where a loop is the plainest statement.

Sources, cited by page title and section:

* "DDTree Deep Dive: Algorithm, Code, and Engineering Philosophy of Block
  Diffusion Draft Trees" (zhichai.net forum post; below: *Deep Dive*):
  §1 per-position marginals and the factorized surrogate Q(y)=prod q_i(y_i);
  §2 Proposition 1 (additivity), Proposition 2 (the top-B prefixes form an
  optimal prefix-closed tree), Lemma 1 (top-K with K=min(B,|V|) suffices),
  Proposition 3 (best-first heap over rank tuples: pop the best, push its
  next sibling and its first child); §3 tree_indices = [position, parent];
  §4 ancestor-only mask; §5 KV-cache compaction; §6 verifier walk.
* "DDTree: Turning Block Diffusion Drafters into Tree-Based Speculative
  Decoders" (alanhou.org; below: *Block Diffusion Drafters*): Core Mechanism
  (score = cumulative log-probability; longest matching prefix accepted) and
  Key Concepts (node D attends to root, A, D only).
* "Qwen3-Coder-30B-A3B · DDTree vs DFlash vs autoregressive" (autobench
  config page): the tree mask is what forces the pages' verifier onto a
  dense masked attention (torch SDPA with a custom mask).

Readings where the pages leave a step open (each one is listed again in the
design notes):

R1  Top-K ranks tokens on the raw logit, descending, lower token id first on
    equal values; -0.0 equals +0.0; NaN is rejected.  (Ranking on z or on
    log q gives the same order in exact arithmetic.)
R2  log q_i is computed in float64 and rounded once to float32; the tree is
    built from that float32 table.
R3  A prefix's score is its log-value log q(u) accumulated in float32 in
    root-to-leaf order, one correctly rounded add per depth.
R4  Total order on prefixes: score descending, then rank tuple
    lexicographically ascending (a proper prefix before its extensions).
R5  B counts non-root nodes; node 0 is the root (the bonus token); nodes
    1..n-1 are numbered in pop order, so parent[i] < i.
R6  The whole committed prefix is visible to every tree node; no causal
    mask inside the prefix; Q and K are already rotated.
R7  Greedy verification (temperature 0): the target's argmax takes the
    lowest token id among equal maxima.  accept_len counts the accepted
    draft nodes plus the new bonus token (k + 1).
R9  Adaptive budget: a node is worth adding while its gain q(u) exceeds the
    cost c of verifying one more node (in accepted tokens); the build keeps
    the pops whose score is strictly above log c.
R11 Rotary positions: the verify layer turns the tree nodes' Q and K at
    position P + depth with the half-split RoPE pairing and base theta
    (1e6 for the Qwen3 family the pages use; a parameter).
R10 Temperature T > 0: the verifier draws the target's token at every tree
    node from softmax(z / T) and walks as at temperature 0; each committed
    token is then a draw from the target at its context, so the output
    follows the target distribution (Deep Dive §6 and §9 assert this property
    and give no rule).  The draws use Philox4x64-10 uniforms and the
    Gumbel-max identity (sample_rows).
"""
from __future__ import annotations

import dataclasses
import heapq
import itertools
from typing import List, Optional, Sequence, Tuple

import numpy as np

PAGE = 64


# --------------------------------------------------------------------------
# Stage 1: per-position log-softmax and top-K
# --------------------------------------------------------------------------

def log_softmax(z: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """log q_i = z_i - logsumexp(z_i) along the last axis, in float64.

    Deep Dive §1: one drafter pass gives per-position marginals q_1..q_L; the
    tree is scored with their logarithms (Block Diffusion Drafters, Core
    Mechanism: cumulative log-probability).  Returns (lp, lse) in float64.
    """
    z = np.asarray(z, dtype=np.float64)
    if np.isnan(z).any():
        raise ValueError("NaN logits are not a valid drafter output")
    m = np.max(z, axis=-1, keepdims=True)
    s = np.sum(np.exp(z - m), axis=-1, keepdims=True)
    lse = m + np.log(s)
    return z - lse, lse[..., 0]


def topk(z: np.ndarray, K: int):
    """Top-K tokens of every row of ``z`` (shape [..., V]) under reading R1.

    Deep Dive §2, Lemma 1: only the K = min(B, |V|) best tokens of each
    position can appear in an optimal tree.

    Returns ids (int32 [..., K], best first), lp32 (float32 [..., K]: log q of
    those tokens rounded once to float32, reading R2), lse32 (float32 [...])
    and lp64 (float64 [..., V], the full log-softmax).
    """
    z = np.asarray(z, dtype=np.float64)
    V = z.shape[-1]
    if not 1 <= K <= V:
        raise ValueError("need 1 <= K <= V")
    lp64, lse64 = log_softmax(z)
    flat = z.reshape(-1, V)
    ids = np.empty((flat.shape[0], K), dtype=np.int32)
    token = np.arange(V)
    for r in range(flat.shape[0]):
        key = flat[r] + 0.0          # -0.0 + 0.0 == +0.0
        # np.lexsort sorts by the last key first: value descending, id ascending.
        order = np.lexsort((token, -key))
        ids[r] = order[:K]
    ids = ids.reshape(z.shape[:-1] + (K,))
    lp_sel = np.take_along_axis(lp64, ids.astype(np.int64), axis=-1)
    return ids, lp_sel.astype(np.float32), lse64.astype(np.float32), lp64


# --------------------------------------------------------------------------
# Stage 2: best-first heap over rank tuples
# --------------------------------------------------------------------------

@dataclasses.dataclass
class Tree:
    """One request's draft tree, n = B+1 rows (unused rows hold -1 / -inf / 0)."""
    node_token: np.ndarray   # int32 [n]
    parent: np.ndarray       # int32 [n], root -1
    depth: np.ndarray        # int32 [n], root 0
    node_rank: np.ndarray    # int32 [n], rank of the token in its position's top-K; root -1
    score: np.ndarray        # float32 [n], reading R3; root 0
    anc: np.ndarray          # uint32 [n, W] ancestor-or-self bitmask
    n_nodes: int
    tuples: List[Tuple[int, ...]]   # rank tuple of every live node (root: ())

    @property
    def n(self) -> int:
        return int(self.parent.shape[0])


def _empty_tree(B: int) -> Tree:
    n = B + 1
    W = (n + 31) // 32
    return Tree(np.full(n, -1, np.int32), np.full(n, -1, np.int32),
                np.full(n, -1, np.int32), np.full(n, -1, np.int32),
                np.full(n, -np.inf, np.float32), np.zeros((n, W), np.uint32), 0, [])


def _order_key(score: np.float32, tup: Tuple[int, ...]):
    """Reading R4 as a Python sort key: larger score first, then smaller tuple."""
    return (-float(score), tup)


def build_tree(ids: np.ndarray, lp32: np.ndarray, root_token: int, B: int,
               gain_floor: Optional[float] = None) -> Tree:
    """Top-B prefixes by best-first search (Deep Dive §2, Proposition 3).

    ``ids`` and ``lp32`` are one request's [L, K] top-K table.  The frontier
    starts with the best token of position 1.  Each step pops the frontier's
    best entry (reading R4), makes it the next node, and pushes its next
    sibling (same parent, rank + 1) and its first child (one position deeper,
    rank 0).  Proposition 2 says the B popped prefixes are the top-B set and
    form a prefix-closed tree.

    ``gain_floor`` (reading R9, the adaptive budget of Deep Dive §10): a pop
    adds q(u) = exp(score) to the expected acceptance (Proposition 1), so
    popping stops at the first pop whose float32 score is not strictly above
    ``gain_floor`` = log c, c being the verification cost of one more node in
    accepted tokens; that pop is not kept.  A NaN floor keeps nothing.
    """
    L, K = lp32.shape
    t = _empty_tree(B)
    t.node_token[0] = root_token
    t.depth[0] = 0
    t.score[0] = np.float32(0.0)
    t.tuples = [()]
    floor = None if gain_floor is None else np.float32(gain_floor)
    # heap entries: (order key, parent node, depth d (1-based), rank r, score)
    heap = []
    s0 = np.float32(np.float32(0.0) + lp32[0, 0])
    heapq.heappush(heap, (_order_key(s0, (0,)), 0, 1, 0, s0))
    pops = 0
    while pops < B and heap:
        (_, tup), par, d, r, s = heapq.heappop(heap)
        if floor is not None and not (s > floor):
            break
        pops += 1
        node = pops
        t.node_token[node] = ids[d - 1, r]
        t.parent[node] = par
        t.depth[node] = d
        t.node_rank[node] = r
        t.score[node] = s
        t.tuples.append(tup)
        if r + 1 < K:   # next sibling: same parent, next rank at this depth
            ss = np.float32(t.score[par] + lp32[d - 1, r + 1])
            heapq.heappush(heap, (_order_key(ss, tup[:-1] + (r + 1,)), par, d, r + 1, ss))
        if d < L:       # first child: one position deeper, rank 0
            sc = np.float32(s + lp32[d, 0])
            heapq.heappush(heap, (_order_key(sc, tup + (0,)), node, d + 1, 0, sc))
    t.n_nodes = pops + 1
    t.anc = ancestor_mask(t.parent, t.n_nodes, B + 1)
    return t


def ancestor_mask(parent: np.ndarray, n_nodes: int, n: int) -> np.ndarray:
    """anc[i] = anc[parent[i]] | {i}: the ancestor-or-self set of every node.

    Deep Dive §4: a node sees the committed context, the root, its ancestors
    and itself, never a sibling or another branch.  Bit j of row i is bit
    (j % 32) of word j // 32.
    """
    W = (n + 31) // 32
    anc = np.zeros((n, W), dtype=np.uint32)
    for i in range(n_nodes):
        if i > 0:
            anc[i] = anc[parent[i]]
        anc[i, i // 32] |= np.uint32(1 << (i % 32))
    return anc


def build_trees(ids: np.ndarray, lp32: np.ndarray, root_token: Sequence[int], B: int,
                gain_floor: Optional[Sequence[float]] = None) -> List[Tree]:
    """``build_tree`` for each request of an [N, L, K] table."""
    return [build_tree(ids[r], lp32[r], int(root_token[r]), B,
                       None if gain_floor is None else float(gain_floor[r])) for r in range(ids.shape[0])]


def stack_trees(trees: List[Tree]):
    """Stack per-request trees into the [N, n] / [N, n, W] arrays of the C ABI."""
    return dict(
        node_token=np.stack([t.node_token for t in trees]),
        parent=np.stack([t.parent for t in trees]),
        depth=np.stack([t.depth for t in trees]),
        node_rank=np.stack([t.node_rank for t in trees]),
        score=np.stack([t.score for t in trees]),
        anc=np.stack([t.anc for t in trees]),
        n_nodes=np.array([t.n_nodes for t in trees], dtype=np.int32),
    )


def prefix_score(lp32: np.ndarray, tup: Tuple[int, ...]) -> np.float32:
    """Reading R3: fp32 sum of the tuple's log-probs in root-to-leaf order."""
    s = np.float32(0.0)
    for d, r in enumerate(tup):
        s = np.float32(s + lp32[d, r])
    return s


def bruteforce_top_prefixes(lp32: np.ndarray, B: int) -> List[Tuple[int, ...]]:
    """All sum_{d<=L} K^d prefixes sorted by reading R4; the first B.

    The exhaustive search that Deep Dive §2 contrasts with the heap
    (O(K^L)); Proposition 2 says its first B entries are the optimal tree.
    """
    L, K = lp32.shape
    allp = []
    for d in range(1, L + 1):
        for tup in itertools.product(range(K), repeat=d):
            allp.append((_order_key(prefix_score(lp32, tup), tup), tup))
    allp.sort()
    return [tup for _, tup in allp[:B]]


def beam_tree(lp32: np.ndarray, width: int) -> List[Tuple[int, ...]]:
    """Beam search tree (Deep Dive §2 and §7: the local heuristic).

    Depth by depth, every kept prefix is extended by all K ranks and the
    ``width`` best extensions (reading R4) are kept.  The tree is the union
    of the beams of all depths.
    """
    L, K = lp32.shape
    beam = [()]
    tree = []
    for _ in range(L):
        cand = [(_order_key(prefix_score(lp32, u + (r,)), u + (r,)), u + (r,))
                for u in beam for r in range(K)]
        cand.sort()
        beam = [u for _, u in cand[:width]]
        tree.extend(beam)
    return tree


def chain_tree(L: int) -> List[Tuple[int, ...]]:
    """The single drafted line (argmax of every position): Deep Dive §1."""
    return [tuple([0] * d) for d in range(1, L + 1)]


def surrogate_value(tuples: Sequence[Tuple[int, ...]], lp64_topk: np.ndarray) -> float:
    """sum_{u in T} q(u) with q(u) = prod_{i<=|u|} q_i(u_i) (Deep Dive §1-§2)."""
    total = 0.0
    for tup in tuples:
        if len(tup) == 0:
            continue
        q = 1.0
        for d, r in enumerate(tup):
            q *= float(np.exp(lp64_topk[d, r]))
        total += q
    return total


def expected_acceptance_enumerated(tree: Tree, p_topk: np.ndarray) -> float:
    """E_{Y~Q}[alpha_T(Y)] by enumerating every draw (Deep Dive §2, Prop. 1).

    ``p_topk`` is [L, K]: the probabilities of each position's top-K tokens.
    Every token outside the top-K is one outcome "other" (index K) with the
    remaining mass; such a draw leaves the tree.  alpha_T(Y) counts the depths
    d whose prefix Y_1:d is a node of T.  The walk down the tree uses the
    parent and rank arrays, not the node tuples.
    """
    L, K = p_topk.shape
    other = 1.0 - p_topk.sum(axis=1)
    child = {}
    for i in range(1, tree.n_nodes):
        child[(int(tree.parent[i]), int(tree.node_rank[i]))] = i
    total = 0.0
    for draw in itertools.product(range(K + 1), repeat=L):
        w = 1.0
        for d, r in enumerate(draw):
            w *= other[d] if r == K else p_topk[d, r]
        if w == 0.0:
            continue
        cur, alpha = 0, 0
        for r in draw:
            nxt = child.get((cur, r)) if r < K else None
            if nxt is None:
                break
            alpha += 1
            cur = nxt
        total += w * alpha
    return total


# --------------------------------------------------------------------------
# Stage 3: ancestor-only tree attention
# --------------------------------------------------------------------------

def _slot_rows(cache: np.ndarray, layer: int, req: int, slots: np.ndarray,
               block_table: Optional[np.ndarray]) -> np.ndarray:
    """Rows [len(slots), Hkv, D] of one request's cache at logical slots."""
    if block_table is None:
        return cache[layer, req, slots]
    blocks = block_table[req, slots // PAGE]
    return cache[layer, blocks, slots % PAGE]


def tree_attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                   prefix_len: np.ndarray, anc: np.ndarray, n_nodes: np.ndarray,
                   scale: float, block_table: Optional[np.ndarray] = None,
                   layers: Optional[Sequence[int]] = None,
                   reqs: Optional[Sequence[int]] = None,
                   heads: Optional[Sequence[int]] = None,
                   nodes: Optional[Sequence[int]] = None):
    """Dense masked attention of the tree nodes, in float64.

    Deep Dive §4: node i of request r attends to the committed prefix
    (slots 0..P_r-1, reading R6) and to the tree slots P_r + j of every j in
    its ancestor-or-self set (bit j of ``anc[r, i]``); query head h reads KV
    head h // (Hq / Hkv).  s = (q . k) * scale, p = softmax(s), o = p . v.

    q: [layers, N, n, Hq, D]; caches contiguous [layers, N, S, Hkv, D] or
    paged [layers, blocks, 64, Hkv, D] with ``block_table`` [N, max_blocks].
    Optional index lists restrict the work to a sample.  Returns a dict
    mapping (layer, req, node, head) -> float64 [D] output row, and the
    float64 natural-log sum-exp of that row's scores.
    """
    nl, N, n, Hq, D = q.shape
    Hkv = k_cache.shape[-2]
    G = Hq // Hkv
    layers = range(nl) if layers is None else layers
    reqs = range(N) if reqs is None else reqs
    heads = range(Hq) if heads is None else heads
    out, lse = {}, {}
    for l in layers:
        for r in reqs:
            P = int(prefix_len[r])
            nn = int(n_nodes[r])
            node_list = range(nn) if nodes is None else [i for i in nodes if i < nn]
            pre_slots = np.arange(P)
            tree_slots = P + np.arange(nn)
            Kp = _slot_rows(k_cache, l, r, pre_slots, block_table).astype(np.float64)
            Vp = _slot_rows(v_cache, l, r, pre_slots, block_table).astype(np.float64)
            Kt = _slot_rows(k_cache, l, r, tree_slots, block_table).astype(np.float64)
            Vt = _slot_rows(v_cache, l, r, tree_slots, block_table).astype(np.float64)
            for i in node_list:
                vis = np.array([(int(anc[r, i, j // 32]) >> (j % 32)) & 1 for j in range(nn)],
                               dtype=bool)
                for h in heads:
                    g = h // G
                    qv = q[l, r, i, h].astype(np.float64)
                    keys = np.concatenate([Kp[:, g], Kt[vis, g]], axis=0)
                    vals = np.concatenate([Vp[:, g], Vt[vis, g]], axis=0)
                    s = (keys @ qv) * scale
                    m = s.max()
                    e = np.exp(s - m)
                    out[(l, r, i, h)] = (e @ vals) / e.sum()
                    lse[(l, r, i, h)] = m + np.log(e.sum())
    return out, lse


# --------------------------------------------------------------------------
# Stage 4: greedy verifier walk and KV compaction
# --------------------------------------------------------------------------

def argmax_rows(x: np.ndarray) -> np.ndarray:
    """Index of the first maximum along the last axis (reading R7)."""
    x = np.asarray(x, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN target logits")
    return np.argmax(x, axis=-1).astype(np.int32)


@dataclasses.dataclass
class Acceptance:
    path: np.ndarray        # int32 [L+1] node ids, path[0] = 0, -1 past accept_len
    accept_len: int         # k + 1
    next_bonus: int         # target argmax at the last accepted node
    src_slot: np.ndarray    # int32 [L+1] P + path[j]
    dst_slot: np.ndarray    # int32 [L+1] P + j
    new_prefix_len: int     # P + k + 1
    target_argmax: np.ndarray


def accept(target: np.ndarray, node_token: np.ndarray, parent: np.ndarray,
           n_nodes: int, L: int, prefix_len: int, tokens: Optional[np.ndarray] = None) -> Acceptance:
    """The verifier walk of Deep Dive §6 for one request.

    Start at the root; while the root-side node has a child whose token is
    the target's token at that node, descend into it.  The first unmatched
    token is the next bonus token (Block Diffusion Drafters, Core Mechanism:
    the longest matching prefix is accepted).  The target's token at a node
    is its argmax at temperature 0 (reading R7), or ``tokens`` when given
    (a draw per node at temperature > 0, reading R10: ``sample_rows``).
    """
    t = argmax_rows(target[:n_nodes]) if tokens is None else np.asarray(tokens[:n_nodes], dtype=np.int64)
    cur = 0
    path = [0]
    while True:
        nxt = None
        for c in range(1, n_nodes):
            if parent[c] == cur and node_token[c] == t[cur]:
                nxt = c
                break
        if nxt is None:
            break
        path.append(nxt)
        cur = nxt
    k = len(path) - 1
    p = np.full(L + 1, -1, np.int32)
    p[:k + 1] = path
    src = np.full(L + 1, -1, np.int32)
    dst = np.full(L + 1, -1, np.int32)
    src[:k + 1] = prefix_len + np.array(path)
    dst[:k + 1] = prefix_len + np.arange(k + 1)
    return Acceptance(p, k + 1, int(t[cur]), src, dst, prefix_len + k + 1, t)


# --------------------------------------------------------------------------
# Tree K/V into the cache with rotary positions (the verify layer's neighbour)
# --------------------------------------------------------------------------

def tree_positions(depth: np.ndarray, prefix_len: int, n_nodes: int) -> np.ndarray:
    """Sequence position of every live node: P + depth (Deep Dive §3,
    tree_compile: a node's position id is its depth past the committed
    prefix)."""
    return prefix_len + np.asarray(depth[:n_nodes], dtype=np.int64)


def rope(x: np.ndarray, pos: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding (Su et al., "RoFormer", §3.4), half-split
    pairing (reading R11): for i < D/2, the pair (x_i, x_{i+D/2}) turns by the
    angle pos * theta^(-2i/D).  ``x`` is [..., D] with the position axis
    leading (``pos`` broadcasts over the middle axes); float64."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    h = D // 2
    inv = theta ** (-(2.0 * np.arange(h)) / D)
    ang = np.asarray(pos, dtype=np.float64).reshape((-1,) + (1,) * (x.ndim - 1)) * inv
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def write_tree_kv(k_cache: np.ndarray, v_cache: np.ndarray, k_in: np.ndarray, v_in: np.ndarray,
                  depth: np.ndarray, prefix_len: np.ndarray, n_nodes: np.ndarray, theta: float,
                  block_table: Optional[np.ndarray] = None) -> None:
    """The tree nodes' K and V into their cache slots (Deep Dive §5: tree
    K/V sit in the cache tail, node i at slot P + i): K rotated at position
    P + depth[i], V as is.  k_in / v_in are [layers, N, n, Hkv, D]; the caches
    are contiguous [layers, N, S, Hkv, D] or paged pools with ``block_table``;
    writes float64 values into them (the caller rounds)."""
    layers, N = k_in.shape[0], k_in.shape[1]
    for r in range(N):
        nn = int(n_nodes[r])
        P = int(prefix_len[r])
        pos = tree_positions(depth[r], P, nn)
        slots = P + np.arange(nn)
        for l in range(layers):
            kr = rope(k_in[l, r, :nn], pos, theta) if theta > 0 else np.asarray(k_in[l, r, :nn], np.float64)
            vr = np.asarray(v_in[l, r, :nn], np.float64)
            if block_table is None:
                k_cache[l, r, slots] = kr
                v_cache[l, r, slots] = vr
            else:
                blk = block_table[r, slots // PAGE]
                k_cache[l, blk, slots % PAGE] = kr
                v_cache[l, blk, slots % PAGE] = vr


def lm_head_argmax(hidden: np.ndarray, weight: np.ndarray):
    """The target's token at each node from its LM head (Deep Dive §6, the
    verifier's argmax): logits = hidden . weight^T in float64, then the
    lowest index among the maxima of each row (reading R7).  Returns (argmax
    int32 [rows], max float64 [rows])."""
    logits = np.asarray(hidden, dtype=np.float64) @ np.asarray(weight, dtype=np.float64).T
    return argmax_rows(logits), logits.max(axis=-1)


# --------------------------------------------------------------------------
# Temperature > 0: one draw of the target's token per tree node
# --------------------------------------------------------------------------

_PHILOX_M = (0xD2E7470EE14C6C93, 0xCA5A826395121157)
_PHILOX_W = (0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B)
_LO32 = np.uint64(0xFFFFFFFF)


def _mulhilo64(a: np.ndarray, b: int):
    """(high, low) 64-bit halves of the 128-bit products a * b (uint64)."""
    b = np.uint64(b)
    a_lo, a_hi = a & _LO32, a >> np.uint64(32)
    b_lo, b_hi = b & _LO32, b >> np.uint64(32)
    ll, lh, hl, hh = a_lo * b_lo, a_lo * b_hi, a_hi * b_lo, a_hi * b_hi
    mid = (ll >> np.uint64(32)) + (lh & _LO32) + (hl & _LO32)
    hi = hh + (lh >> np.uint64(32)) + (hl >> np.uint64(32)) + (mid >> np.uint64(32))
    return hi, a * b


def philox4x64(counter, key) -> np.ndarray:
    """Philox4x64-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
    as easy as 1, 2, 3", SC 2011): ten rounds of two 64x64 -> 128-bit
    multiplications by the published multipliers, a Weyl-sequence key bump
    between rounds.  ``counter`` is four uint64 arrays (broadcast), ``key``
    two uint64; returns [4, ...] uint64 outputs."""
    c = [np.asarray(x, dtype=np.uint64) for x in np.broadcast_arrays(*counter)]
    k0, k1 = int(key[0]) & (2 ** 64 - 1), int(key[1]) & (2 ** 64 - 1)
    with np.errstate(over="ignore"):
        for _ in range(10):
            hi0, lo0 = _mulhilo64(c[0], _PHILOX_M[0])
            hi1, lo1 = _mulhilo64(c[2], _PHILOX_M[1])
            c = [hi1 ^ c[1] ^ np.uint64(k0), lo1, hi0 ^ c[3] ^ np.uint64(k1), lo0]
            k0 = (k0 + _PHILOX_W[0]) & (2 ** 64 - 1)
            k1 = (k1 + _PHILOX_W[1]) & (2 ** 64 - 1)
    return np.stack(c)


def uniforms(V: int, node: int, req: int, seed: int, offset: int) -> np.ndarray:
    """u_v in (0, 1), float64, for v < V: output word v % 4 of Philox4x64-10
    at counter (v // 4, node, req, 0) with key (seed, offset); the top 52
    bits plus one half, times 2^-52 (every step exact in float64)."""
    blocks = (V + 3) // 4
    out = philox4x64((np.arange(blocks, dtype=np.uint64), node, req, 0), (seed, offset))
    words = out.T.reshape(-1)[:V]
    return ((words >> np.uint64(12)).astype(np.float64) + 0.5) * 2.0 ** -52


def sample_rows(target: np.ndarray, temperature: float, seed: int, offset: int, req: int) -> np.ndarray:
    """One draw from softmax(z / temperature) per row (reading R10).

    Gumbel-max: token = argmax_v (z_v / T + g_v), g_v = -log(-log u_v),
    which is a draw from softmax(z / T) (the Gumbel-max identity).  The
    perturbed score is formed in float64 (z times the float64 value of 1/T)
    and rounded once to float32; the argmax takes the lowest token id among
    equal maxima, like the temperature-0 argmax.  NaN logits are rejected.
    """
    x = np.asarray(target, dtype=np.float64)
    if np.isnan(x).any():
        raise ValueError("NaN target logits")
    inv_t = 1.0 / float(temperature)
    out = np.empty(x.shape[0], dtype=np.int32)
    for i in range(x.shape[0]):
        u = uniforms(x.shape[1], i, req, seed, offset)
        g = -np.log(-np.log(u))
        s32 = (x[i] * inv_t + g).astype(np.float32)
        out[i] = int(np.argmax(s32))
    return out


def compact(k_cache: np.ndarray, v_cache: np.ndarray, req: int, acc: Acceptance,
            block_table: Optional[np.ndarray] = None) -> None:
    """In-place KV compaction of the accepted path (Deep Dive §5).

    For every layer, in forward order j = 0..k, the K and V rows of slot
    P + path[j] move to slot P + j.  Forward order is safe in place because
    path[j] >= j and the path increases.
    """
    for j in range(acc.accept_len):
        s, d = int(acc.src_slot[j]), int(acc.dst_slot[j])
        for cache in (k_cache, v_cache):
            if block_table is None:
                cache[:, req, d] = cache[:, req, s]
            else:
                cache[:, block_table[req, d // PAGE], d % PAGE] = \
                    cache[:, block_table[req, s // PAGE], s % PAGE]
