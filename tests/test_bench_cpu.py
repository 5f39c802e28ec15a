"""Host logic of bench.py (no GPU): the algorithmic work model, the stage
roof fractions and the source-keyed traffic table."""
import types

import numpy as np
import pytest
import torch

import bench
from draft_tree_build_ddtree_b200 import datagen


def _fake_round(w, n_nodes, anc_bits, prefix, accept_len):
    """A stand-in for RoundBuffers holding only what algorithmic_work reads."""
    N, n, W = w.N, w.n, w.W
    anc = np.zeros((N, n, W), dtype=np.uint32)
    for r in range(N):
        for i, bits in enumerate(anc_bits[r]):
            for j in bits:
                anc[r, i, j // 32] |= np.uint32(1 << (j % 32))
    tree = types.SimpleNamespace(n_nodes=torch.tensor(n_nodes, dtype=torch.int32),
                                 anc=torch.from_numpy(anc.view(np.int32)))
    acc = types.SimpleNamespace(accept_len=torch.tensor(accept_len, dtype=torch.int32))
    return types.SimpleNamespace(tree=tree, prefix_len=torch.tensor(prefix, dtype=torch.int32), acc=acc)


def test_algorithmic_work_follows_its_definition():
    w = datagen.workload(1)              # fp32, N=1, L=4, V=512, K=8, B=16, Hq=2, Hkv=1, D=64, P=128
    # a 4-node chain 0 <- 1 <- 2 <- 3: node i sees nodes 0..i
    rows = [[list(range(i + 1)) for i in range(4)]]
    rb = _fake_round(w, [4], rows, [w.P], [3])
    work = bench.algorithmic_work(w, rb)
    es = 4
    assert work["topk"]["bytes"] == w.N * w.L * w.V * es + w.N * w.L * (w.K * 8 + 4)
    visible = 1 + 2 + 3 + 4
    assert work["attn"]["flops"] == w.layers * 4 * w.Hq * w.D * (4 * w.P + visible)
    assert work["attn"]["bytes"] == w.layers * ((w.P + 4) * w.Hkv * w.D * es * 2 + 2 * 4 * w.Hq * w.D * es)
    # argmax over the live rows, then 2 accepted rows moved for K and V (read + write) per layer
    assert work["accept"]["bytes"] == 4 * w.V * es + 2 * 2 * 2 * w.layers * w.Hkv * w.D * es


def test_stage_report_bound_and_fraction():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0, "bf16_tflops_sustained": 80.0}
    work = {"topk": {"bytes": 2e9, "flops": 0},
            "build": {"bytes": 1e6, "flops": 0},
            "attn": {"bytes": 1e9, "flops": 1e12},      # 1000 flop/B > ridge 100 flop/B: tensor-bound
            "accept": {"bytes": 5e8, "flops": 0}}
    stage_ms = {"topk": 4.0, "build": 1.0, "attn": 20.0, "accept": 1.0}
    st, tp = bench.stage_report(None, work, stage_ms, peaks, long_region=False)
    assert tp == 100.0
    assert st["topk"]["bound"] == "hbm" and st["topk"]["frac"] == pytest.approx(0.5)         # 500 GB/s of 1000
    assert st["topk"]["hbm_frac_nominal"] == pytest.approx(500.0 / bench.NOMINAL_HBM_GBS)
    assert st["build"]["bound"] == "latency"
    assert st["attn"]["bound"] == "tensor" and st["attn"]["frac"] == pytest.approx(0.5)     # 50 TFLOP/s of 100
    assert st["attn"]["tensor_frac_sustained"] == pytest.approx(50.0 / 80.0)
    st2, tp2 = bench.stage_report(None, work, stage_ms, peaks, long_region=True)
    assert tp2 == 80.0 and st2["attn"]["frac"] == pytest.approx(50.0 / 80.0)


def test_traffic_table_reads_null_once_the_sources_change(monkeypatch):
    files = ("topk.cuh", "common.cuh")
    good = bench.sources_digest(files)
    monkeypatch.setattr(bench, "TRAFFIC", {("w", "topk"): (123, files, good), ("w", "attn"): (456, files, "0" * 16)})
    assert bench.measured_traffic("w", "topk") == 123
    assert bench.measured_traffic("w", "attn") is None       # digest of other sources
    assert bench.measured_traffic("other", "topk") is None   # no capture for this workload
