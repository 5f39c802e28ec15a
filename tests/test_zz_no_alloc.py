"""GPU test of ddtree_topk_static_ws, the top-K entry point with built-in scratch.

Some callers cannot allocate device memory while they run rounds: a serving
engine that gives all free device memory to its KV-cache pool at start-up
must not call cudaMalloc at decode time, where it can synchronize the device
or fail because the pool already holds the memory.  For them the library has
a top-K call that uses a fixed scratch array built into the library instead
of a caller workspace.  This test calls it through the C ABI and checks that
it returns what ddtree_topk returns on the same logits, on two calls in a
row (the second call reuses the array the first one left behind).

The file name sorts last so that a run that stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import draft_tree_build_ddtree_b200 as dd
from draft_tree_build_ddtree_b200 import datagen

pytestmark = pytest.mark.gpu
CUDA = "cuda:0"
LP_TOL = 1e-5


def _static_topk(logits: torch.Tensor, K: int):
    rows, V = logits.shape
    ids = torch.full((rows, K), -1, dtype=torch.int32, device=CUDA)
    lp = torch.full((rows, K), float("nan"), dtype=torch.float32, device=CUDA)
    lse = torch.full((rows,), float("nan"), dtype=torch.float32, device=CUDA)
    dtype = dd.BF16 if logits.dtype == torch.bfloat16 else dd.F32
    st = dd.lib().ddtree_topk_static_ws(ctypes.c_void_p(logits.data_ptr()), dtype, rows, V, logits.stride(0), K,
                                        ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(lp.data_ptr()),
                                        ctypes.c_void_p(lse.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dd.lib().ddtree_status_string(st).decode()
    torch.cuda.synchronize()
    return ids, lp, lse


@pytest.mark.parametrize("cfg", [1, 2])
def test_static_scratch_topk_matches_workspace_topk(cfg):
    w = datagen.workload(cfg)
    x = datagen.drafter_logits(w).reshape(-1, w.V).to(CUDA)
    ref_ids, ref_lp, ref_lse = dd.ddtree_topk(x, w.K)
    torch.cuda.synchronize()
    for _ in range(2):
        ids, lp, lse = _static_topk(x, w.K)
        assert torch.equal(ids, ref_ids)
        assert float((lp - ref_lp).abs().max()) <= LP_TOL
        assert float((lse - ref_lse).abs().max()) <= 4 * LP_TOL
    assert dd.device_status() == 0


def test_static_scratch_rejects_requests_beyond_its_size():
    V, K = 151936, 1024
    x = torch.zeros((64, V), dtype=torch.bfloat16, device=CUDA)
    ids = torch.empty((64, K), dtype=torch.int32, device=CUDA)
    lp = torch.empty((64, K), dtype=torch.float32, device=CUDA)
    st = dd.lib().ddtree_topk_static_ws(ctypes.c_void_p(x.data_ptr()), dd.BF16, 64, V, V, K,
                                        ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(lp.data_ptr()), None,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 7
    assert b"scratch" in dd.lib().ddtree_status_string(st)


def test_static_scratch_largest_accepted_request_and_no_allocation():
    """The largest request the 4 MiB scratch accepts (found through the call
    itself: a rejected request launches nothing) runs like ddtree_topk and the
    oracle on sampled rows; one row more is rejected; and a call after the
    first leaves the device's free memory unchanged."""
    import oracle
    V, K = 151936, 64
    g = torch.Generator().manual_seed(11)
    big = (torch.randn(640, V, generator=g) * 4).to(torch.bfloat16).to(CUDA)
    lo, hi = 1, 640                      # largest accepted row count in [lo, hi)
    while hi - lo > 1:
        mid = (lo + hi) // 2
        ids = torch.empty((mid, K), dtype=torch.int32, device=CUDA)
        lp = torch.empty((mid, K), dtype=torch.float32, device=CUDA)
        st = dd.lib().ddtree_topk_static_ws(ctypes.c_void_p(big.data_ptr()), dd.BF16, mid, V, V, K,
                                            ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(lp.data_ptr()), None,
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st in (0, 7)
        lo, hi = (mid, hi) if st == 0 else (lo, mid)
    rows = lo
    assert 500 <= rows < 640, rows     # about 571 rows on a 148-SM B200
    x = big[:rows]
    ref_ids, ref_lp, ref_lse = dd.ddtree_topk(x, K)
    torch.cuda.synchronize()
    ids, lp, lse = _static_topk(x, K)
    free0 = torch.cuda.mem_get_info()[0]
    ids2, lp2, lse2 = _static_topk(x, K)
    free1 = torch.cuda.mem_get_info()[0]
    assert free1 == free0
    for a, b in ((ids, ref_ids), (ids2, ref_ids)):
        assert torch.equal(a, b)
    assert float((lp2 - ref_lp).abs().max()) <= LP_TOL
    sample = [0, 1, rows // 2, rows - 1]
    o_ids, o_lp, _, _ = oracle.topk(x[sample].to("cpu", torch.float64).numpy(), K)
    assert np.array_equal(ids2[sample].cpu().numpy(), o_ids)
    assert np.max(np.abs(lp2[sample].cpu().numpy().astype(np.float64) - o_lp)) <= LP_TOL
    one_more = torch.empty((rows + 1, K), dtype=torch.int32, device=CUDA)
    lp_more = torch.empty((rows + 1, K), dtype=torch.float32, device=CUDA)
    st = dd.lib().ddtree_topk_static_ws(ctypes.c_void_p(big.data_ptr()), dd.BF16, rows + 1, V, V, K,
                                        ctypes.c_void_p(one_more.data_ptr()), ctypes.c_void_p(lp_more.data_ptr()),
                                        None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 7
    assert dd.device_status() == 0
