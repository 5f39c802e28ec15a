"""GPU parity: top-K/log-softmax and tree build against the oracle.

The build stage is fed the oracle's fp32 log-prob table (and ids), so every
tree array is compared bit for bit.
"""
import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
import oracle
from draft_tree_build_ddtree_b200 import datagen

from parity import assert_topk, assert_tree, oracle_topk, oracle_trees, tree_inputs

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"


def _gpu_topk(z: torch.Tensor, K: int):
    x = z.reshape(-1, z.shape[-1]).to(CUDA)
    ids, lp, lse = dd.ddtree_topk(x, K)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    return ids, lp, lse


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_topk_configs(cfg):
    w = datagen.workload(cfg)
    z = datagen.drafter_logits(w)
    if cfg == 4:
        z = z[:4]
    ids, lp32, lse32 = oracle_topk(z, w.K)
    g = _gpu_topk(z, w.K)
    assert_topk(*g, ids.reshape(-1, w.K), lp32.reshape(-1, w.K), lse32.reshape(-1))
    # fp64 log-sum-exp: the fp32 log-probs round like the oracle's, bit for bit
    assert np.array_equal(g[1].cpu().numpy().view(np.uint32), lp32.reshape(-1, w.K).view(np.uint32))


@pytest.mark.parametrize("sigma", [1.0, 8.0])
def test_topk_k1024_sweep(sigma):
    w = datagen.workload(5, B=1024, sigma=sigma)
    z = datagen.drafter_logits(w)
    ids, lp32, lse32 = oracle_topk(z, w.K)
    g = _gpu_topk(z, w.K)
    assert_topk(*g, ids.reshape(-1, w.K), lp32.reshape(-1, w.K), lse32.reshape(-1))


@pytest.mark.parametrize("V,K,dtype", [(5000, 64, torch.bfloat16), (5000, 1024, torch.bfloat16),
                                       (3000, 100, torch.float32), (151936, 256, torch.bfloat16)])
def test_topk_heavy_ties(V, K, dtype):
    g = torch.Generator().manual_seed(V + K)
    z = torch.randint(-3, 4, (6, V), generator=g).to(dtype)
    z[0, 5] = -0.0
    z[0, 6] = 0.0
    z[1, :100] = float("-inf")
    ids, lp32, lse32 = oracle_topk(z, K)
    assert_topk(*_gpu_topk(z, K), ids, lp32, lse32)


def test_topk_dominant_token_uses_fallback_select():
    # one logit far above the rest: the max-anchored window holds < K values
    g = torch.Generator().manual_seed(4)
    z = torch.randn(4, 151936, generator=g).to(torch.bfloat16)
    z[:, 7] = 300.0
    ids, lp32, lse32 = oracle_topk(z, 64)
    assert_topk(*_gpu_topk(z, 64), ids, lp32, lse32)


@pytest.mark.parametrize("V,K", [(1001, 17), (9, 9), (3, 1)])
def test_topk_ragged_rows(V, K):
    g = torch.Generator().manual_seed(V)
    stride = (V + 7) // 8 * 8
    full = torch.randn(5, stride, generator=g).to(torch.bfloat16)
    ids, lp32, lse32 = oracle_topk(full[:, :V], K)
    x = full.to(CUDA)[:, :V]
    gi, gl, ge = dd.ddtree_topk(x, K)
    assert_topk(gi, gl, ge, ids, lp32, lse32)


def test_topk_many_rows_sampled():
    w = datagen.workload(4)
    z = datagen.drafter_logits(w)            # [32, 16, V]
    gi, gl, ge = _gpu_topk(z, w.K)
    rows = [0, 17, 255, 300, 511]
    flat = z.reshape(-1, w.V)
    ids, lp32, lse32 = oracle_topk(flat[rows], w.K)
    assert_topk(gi[rows], gl[rows], ge[rows], ids, lp32, lse32)


def test_topk_repeat_calls_reuse_workspace():
    w = datagen.workload(2)
    z = datagen.drafter_logits(w)
    a = _gpu_topk(z, w.K)
    b = _gpu_topk(z, w.K)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_topk_nan_sets_status():
    z = torch.randn(2, 4096).to(torch.bfloat16)
    z[1, 100] = float("nan")
    dd.ddtree_topk(z.to(CUDA), 8)
    assert dd.device_status() & dd.STATUS_NONFINITE
    assert dd.device_status() == 0


# ------------------------------------------------------------------ build

def _gpu_build(ids, lp32, root, B):
    t = dd.ddtree_build(torch.from_numpy(np.ascontiguousarray(ids)).to(CUDA),
                        torch.from_numpy(np.ascontiguousarray(lp32)).to(CUDA),
                        torch.from_numpy(np.ascontiguousarray(root).astype(np.int32)).to(CUDA), B)
    torch.cuda.synchronize()
    return t


@pytest.mark.parametrize("cfg", [1, 2, 3])
def test_build_configs(cfg):
    w = datagen.workload(cfg)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    assert_tree(_gpu_build(ids, lp32, root, w.B), st)


@pytest.mark.parametrize("sigma", [1.0, 4.0, 8.0])
def test_build_sweep_b1024(sigma):
    w = datagen.workload(5, B=1024, sigma=sigma)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    assert_tree(_gpu_build(ids, lp32, root, w.B), st)


@pytest.mark.parametrize("B", [16, 128, 512])
def test_build_sweep_budgets(B):
    w = datagen.workload(5, B=B, sigma=4.0)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    assert_tree(_gpu_build(ids, lp32, root, w.B), st)


@pytest.mark.parametrize("seed", range(4))
def test_build_exact_score_ties(seed):
    # coarse tables: many prefixes tie exactly in fp32 and the rank tuple decides
    g = torch.Generator().manual_seed(seed)
    N, L, K, B = 8, 6, 12, 200
    lp = -torch.randint(0, 4, (N, L, K), generator=g).to(torch.float32) * 0.5
    lp = -torch.sort(-lp, dim=-1).values
    ids = torch.randint(0, 1000, (N, L, K), generator=g).to(torch.int32)
    root = torch.arange(N, dtype=torch.int32)
    trees, st = oracle_trees(ids.numpy(), lp.numpy(), root.numpy(), B)
    assert_tree(_gpu_build(ids.numpy(), lp.numpy(), root.numpy(), B), st)


@pytest.mark.parametrize("L,K,B", [(2, 2, 10), (4, 3, 0), (16, 1, 16), (32, 4, 300), (1, 7, 5)])
def test_build_edge_shapes(L, K, B):
    g = torch.Generator().manual_seed(L * 100 + K)
    lp = -torch.rand(3, L, K, generator=g) * 5
    lp = -torch.sort(-lp, dim=-1).values
    ids = torch.randint(0, 5000, (3, L, K), generator=g).to(torch.int32)
    root = torch.tensor([1, 2, 3], dtype=torch.int32)
    trees, st = oracle_trees(ids.numpy(), lp.numpy(), root.numpy(), B)
    assert_tree(_gpu_build(ids.numpy(), lp.numpy(), root.numpy(), B), st)


def test_build_batched_config4():
    w = datagen.workload(4)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    assert_tree(_gpu_build(ids, lp32, root, w.B), st)


# ------------------------------------------------------------------ build: every selection path

def _gpu_build_ex(ids, lp32, root, B, flags=0, floor=None):
    N = ids.shape[0]
    path = torch.full((N,), -7, dtype=torch.int32, device=CUDA)
    fl = None if floor is None else torch.as_tensor(np.asarray(floor, np.float32)).to(CUDA)
    t = dd.ddtree_build(torch.from_numpy(np.ascontiguousarray(ids)).to(CUDA),
                        torch.from_numpy(np.ascontiguousarray(lp32)).to(CUDA),
                        torch.from_numpy(np.ascontiguousarray(root).astype(np.int32)).to(CUDA), B,
                        gain_floor=fl, flags=flags, build_path=path)
    torch.cuda.synchronize()
    return t, path.cpu().numpy()


def _heap_kind(B):
    n = B + 1
    return 1 if n <= 96 else (2 if n <= 288 else 3)


@pytest.mark.parametrize("cfg,over", [(1, {}), (2, {}), (3, {}), (4, {}), (5, dict(B=1024, K=1024)),
                                      (5, dict(B=200, K=200))])
def test_build_forced_heap_matches_oracle(cfg, over):
    """Proposition 3's heap itself (all three queue variants), bit for bit."""
    w = datagen.workload(cfg, **over)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    t, path = _gpu_build_ex(ids, lp32, root, w.B, flags=dd.BUILD_FORCE_HEAP)
    assert np.all(path == _heap_kind(w.B)), path
    assert_tree(t, st)
    # the default call takes the enumeration on these tables and agrees
    t2, path2 = _gpu_build_ex(ids, lp32, root, w.B)
    assert np.all(path2 == 0), path2
    assert_tree(t2, st)


def _tie_table(N, L, K, top_equal, seed):
    """lp tables whose `top_equal` best ranks at every position are exactly
    0.0 (the rest strictly negative): every prefix over those ranks scores
    exactly 0, the largest possible score."""
    g = torch.Generator().manual_seed(seed)
    lp = -(torch.rand(N, L, K, generator=g) * 4 + 0.5)
    lp[:, :, :top_equal] = 0.0
    lp = -torch.sort(-lp, dim=-1).values
    ids = torch.randint(0, 151936, (N, L, K), generator=g).to(torch.int32)
    return ids.numpy(), lp.numpy().astype(np.float32)


@pytest.mark.parametrize("B,K,top_equal", [(64, 64, 64), (95, 8, 8), (200, 64, 4), (287, 16, 16),
                                           (1024, 1024, 1024), (1024, 64, 3)])
def test_build_enumeration_overflow_takes_heap(B, K, top_equal):
    """Tie-heavy tables overflow the enumeration: the kernel reports the heap
    it fell back to, and the tree is the oracle's bit for bit.

    Why the enumeration must overflow, from the oracle's side: the B-th pop
    scores 0, the largest possible score, so any threshold that admits B
    prefixes admits every prefix scoring 0, and there are
    sum_d top_equal^d > 4096 of them."""
    N, L = 3, 16
    ids, lp32 = _tie_table(N, L, K, top_equal, seed=B + K)
    root = np.arange(N, dtype=np.int32)
    trees, st = oracle_trees(ids, lp32, root, B)
    assert np.all(st["score"][:, B] == 0.0)
    assert sum(top_equal ** d for d in range(1, L + 1)) > 4096
    t, path = _gpu_build_ex(ids, lp32, root, B)
    assert np.all(path == _heap_kind(B)), path
    assert_tree(t, st)


@pytest.mark.parametrize("cfg,over", [(1, {}), (2, {}), (3, {}), (5, dict(B=1024, K=1024, sigma=8.0))])
@pytest.mark.parametrize("flags", [0, 1])
def test_build_adaptive_floor_matches_oracle(cfg, over, flags):
    """Adaptive budget (gain floor): the kept pops are the oracle's, bit for
    bit, for floors at a node's exact score, between scores, and the edges."""
    w = datagen.workload(cfg, **over)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    s = st["score"][0]
    nn = int(st["n_nodes"][0])
    cases = [float(s[nn // 2]), float(np.float32(s[nn // 3]) - np.float32(1e-3)), -np.inf, np.inf, np.nan,
             -1e30, 0.0]
    for f in cases:
        floor = np.full(w.N, f, np.float32)
        ref = oracle.stack_trees(oracle.build_trees(ids, lp32, root, w.B, gain_floor=floor))
        t, path = _gpu_build_ex(ids, lp32, root, w.B, flags=flags, floor=floor)
        assert_tree(t, ref)


def test_build_adaptive_floor_per_request():
    """Each request keeps its own floor (batched workload, mixed floors)."""
    w = datagen.workload(4)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    g = np.random.default_rng(5)
    floor = np.array([float(st["score"][r, g.integers(1, w.n)]) for r in range(w.N)], np.float32)
    floor[3] = -np.inf
    floor[7] = np.nan
    ref = oracle.stack_trees(oracle.build_trees(ids, lp32, root, w.B, gain_floor=floor))
    t, _ = _gpu_build_ex(ids, lp32, root, w.B, floor=floor)
    assert_tree(t, ref)
