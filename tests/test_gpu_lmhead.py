"""GPU parity of the LM head with its argmax fused into the product
(ddtree_lmhead_argmax), of the walk from given tokens (ddtree_walk) and of
the round that takes the target's tokens from the LM head, against the
oracle (float64 logits, lowest index among the maxima).

The GPU accumulates in fp32 on the tensor cores in the hardware's order, so
two logits within that rounding of each other may resolve either way: a
differing argmax is accepted only where the oracle's two logits differ by
less than the fp32 accumulation bound, sum_k |h_k w_k| * 2^-20.
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


def _lm_inputs(rows, V, d, seed):
    g = torch.Generator().manual_seed(seed)
    h = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    w = (torch.randn(V, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    return h, w


def _check_argmax(got, h, w, got_max=None):
    h64, w64 = h.to(torch.float64).numpy(), w.to(torch.float64).numpy()
    ref, mx = oracle.lm_head_argmax(h64, w64)
    for r in np.nonzero(got != ref)[0]:
        a, b = int(ref[r]), int(got[r])
        la, lb = h64[r] @ w64[a], h64[r] @ w64[b]
        bound = max(np.abs(h64[r] * w64[a]).sum(), np.abs(h64[r] * w64[b]).sum()) * 2.0 ** -20
        assert abs(la - lb) <= bound, (r, a, b, la, lb, bound)
    if got_max is not None:
        bound = (np.abs(h64) @ np.abs(w64).max(axis=0)) * 2.0 ** -20 + 1e-6
        assert np.all(np.abs(got_max - mx) <= np.maximum(bound, 1e-5 * np.abs(mx)))
    return ref


@pytest.mark.parametrize("rows,V,d", [(65, 151936, 512), (257, 20000, 2048), (300, 4099, 128), (1, 256, 64)])
def test_lmhead_argmax_matches_oracle(rows, V, d):
    h, w = _lm_inputs(rows, V, d, seed=rows + V + d)
    mx = torch.empty(rows, dtype=torch.float32, device=CUDA)
    got = dd.ddtree_lmhead_argmax(h.to(CUDA), w.to(CUDA), out_max=mx)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    _check_argmax(got.cpu().numpy(), h, w, mx.cpu().numpy().astype(np.float64))
    # the workspace is left at zero: a second call gives the same answer
    again = dd.ddtree_lmhead_argmax(h.to(CUDA), w.to(CUDA))
    torch.cuda.synchronize()
    assert torch.equal(got, again)


def test_walk_from_tokens_matches_accept():
    """ddtree_walk on the oracle's argmax tokens equals the greedy accept."""
    w = datagen.workload(2)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    nn = int(st["n_nodes"][0])
    tok = np.full((1, w.n), -1, np.int32)
    tok[0, :nn] = oracle.argmax_rows(tgt[0, :nn].to(torch.float64).numpy())
    kd, vd = cache.k.to(CUDA), cache.v.to(CUDA)
    kv = dd.kv_desc_for(kd, w.N, w.Hq)
    acc = dd.ddtree_walk(torch.from_numpy(tok).to(CUDA), torch.from_numpy(st["node_token"]).to(CUDA),
                         torch.from_numpy(st["parent"]).to(CUDA), torch.from_numpy(st["n_nodes"]).to(CUDA), w.L,
                         prefix.to(CUDA), kd, vd, kv)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    a = oracle.accept(tgt[0].to(torch.float64).numpy(), st["node_token"][0], st["parent"][0], nn, w.L,
                      int(prefix[0]))
    assert acc.path[0].tolist() == a.path.tolist()
    assert int(acc.accept_len[0]) == a.accept_len and int(acc.next_bonus[0]) == a.next_bonus
    kh, vh = raw_bits(cache.k), raw_bits(cache.v)
    oracle.compact(kh, vh, 0, a)
    assert np.array_equal(raw_bits(kd), kh) and np.array_equal(raw_bits(vd), vh)


@pytest.mark.parametrize("cfg,over", [(2, {}), (4, dict(N=3))])
def test_round_with_lm_head(cfg, over):
    """The round takes each node's token from the LM head of the nodes'
    hidden states (logits never materialised) and walks with it."""
    w = datagen.workload(cfg, **over)
    z, ids, lp32, lse32, root, trees, st = tree_inputs(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q = datagen.queries(w)
    d = 512
    h, lm = _lm_inputs(w.N * w.n, w.V, d, seed=77 + cfg)
    tgt_unused = torch.zeros((w.N, w.n, 8), dtype=torch.bfloat16)
    rb = dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B, kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=z.to(CUDA), root_token=torch.from_numpy(root).to(CUDA), q=q.to(CUDA),
        k_cache=cache.k.to(CUDA), v_cache=cache.v.to(CUDA),
        block_table=None if cache.block_table is None else cache.block_table.to(CUDA),
        prefix_len=prefix.to(CUDA), target_logits=tgt_unused.to(CUDA),
        target_hidden=h.to(CUDA), lm_head=lm.to(CUDA)).allocate_outputs()
    assert dd.ddtree_round_launch_count(rb) >= 5
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    assert dd.device_status() == 0
    got = rb.acc.target_argmax.cpu().numpy().reshape(-1)
    tok = _check_argmax(got, h, lm).reshape(w.N, w.n)
    tok = np.where(got.reshape(w.N, w.n) != tok, got.reshape(w.N, w.n), tok)    # accepted near-ties
    kh, vh = raw_bits(cache.k), raw_bits(cache.v)
    table = None if cache.block_table is None else cache.block_table.numpy()
    for r in range(w.N):
        nn = int(st["n_nodes"][r])
        a = oracle.accept(None, st["node_token"][r], st["parent"][r], nn, w.L, int(prefix[r]), tokens=tok[r])
        assert rb.acc.path[r].tolist() == a.path.tolist()
        assert int(rb.acc.next_bonus[r]) == a.next_bonus
        assert int(rb.acc.new_prefix_len[r]) == a.new_prefix_len
        oracle.compact(kh, vh, r, a, block_table=table)
    assert np.array_equal(raw_bits(rb.k_cache), kh) and np.array_equal(raw_bits(rb.v_cache), vh)
