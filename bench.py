#!/usr/bin/env python
"""Benchmark one DDTree draft-and-verify round (ddtree_round) on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one ddtree_round (top-K -> tree build -> tree attention over all
of the workload's layers -> verifier walk + KV compaction) over one batch of
synthetic inputs already resident in HBM.  Steps rotate over enough input
sets that consecutive steps never find their inputs in L2.  Each rank runs
its own independent rounds (replicas: the round of one request batch does
not shard), timed with CUDA events and reduced as the max over ranks; rank
0 prints one JSON line.

``--impl reference`` times the CPU oracle (the checker, plain numpy) on the
host, each step a bounded sample of the same workload, extrapolated to the
same metric.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from draft_tree_build_ddtree_b200 import datagen  # noqa: E402

METRIC = "DDTree rounds/s at 1 B200; tree-attn & top-K % of HBM roofline"
UNIT = "rounds/s"
L2_BYTES = 126 * 1024 * 1024
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--budget", type=int, default=None, help="config 5: B")
    ap.add_argument("--sigma", type=float, default=None, help="config 5: drafter logit std-dev")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch rounds eagerly instead of CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="profiling driver: one input set, warmup + steps eager rounds, no timing")
    return ap.parse_args()


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture, with a hash of the kernel's sources at capture time: the value
# is reported only while the sources are unchanged (summaries under profiles/).
CSRC = os.path.join(os.path.dirname(os.path.abspath(__file__)), "draft_tree_build_ddtree_b200", "csrc")
TRAFFIC = {
    ("b64_p2k", "topk"): (5069568, ("topk.cuh", "common.cuh", "exp64_table.h"), "4c480e2f4cca5119"),
    ("b256_p8k_48l", "attn"): (1057939712, ("attn_tc.cuh", "attn_simt.cuh", "common.cuh"), "673c3d78fa774a8f"),
}


def measured_traffic(workload: str, stage: str):
    import hashlib
    entry = TRAFFIC.get((workload, stage))
    if entry is None:
        return None
    nbytes, files, digest = entry
    m = hashlib.sha256()
    try:
        for f in files:
            with open(os.path.join(CSRC, f), "rb") as fh:
                m.update(fh.read())
    except OSError:
        return None
    return nbytes if m.hexdigest()[:16] == digest else None


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- distributed plumbing

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world: int, backend: str = "nccl"):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the value itself when alone)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and torch.device(device).type == "cuda":
            torch.distributed.barrier(device_ids=[torch.device(device).index])
        else:
            torch.distributed.barrier()


def aggregate_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_rank * world / seconds_max


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-i", str(self.gpu),
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [x for x in sm if mx is None or x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- workload

def workload_from_args(a):
    if a.config == 5:
        return datagen.workload(5, B=a.budget if a.budget else 64, sigma=a.sigma if a.sigma else 4.0)
    return datagen.workload(a.config)


def workload_label(w) -> str:
    """The workload's name and sizes, as both arms report it."""
    return (f"{w.name}: L={w.L} V={w.V} K={w.K} B={w.B} Hq={w.Hq} Hkv={w.Hkv} "
            f"D={w.D} P={w.P or f'U[{w.P_lo},{w.P_hi}]'} layers={w.layers} "
            f"n_req={w.N}{' paged' if w.paged else ''}")


def set_bytes(w) -> int:
    es = 2 if w.dtype == "bf16" else 4
    prefix = datagen.prefix_lengths(w)
    S = datagen.slots_needed(w, prefix)
    kv = 2 * w.layers * w.N * S * w.Hkv * w.D * es
    return (w.N * w.L * w.V + w.N * w.n * w.V) * es + w.layers * w.N * w.n * w.Hq * w.D * es + kv


def make_sets(w, R, device):
    """R independent input sets on the device, each a ready RoundBuffers."""
    import draft_tree_build_ddtree_b200 as dd
    sets = []
    for rep in range(R):
        z = datagen.drafter_logits(w, rep)
        prefix = datagen.prefix_lengths(w, rep)
        cache = datagen.kv_cache(w, prefix, rep)
        q = datagen.queries(w, rep)
        root = datagen.root_tokens(w, rep)
        zd = z.to(device)
        rootd = root.to(device)
        # the target logits follow the tree, which the library builds here
        ids, lp, _ = dd.ddtree_topk(zd.reshape(-1, w.V), w.K)
        tree = dd.ddtree_build(ids.reshape(w.N, w.L, w.K), lp.reshape(w.N, w.L, w.K), rootd, w.B)
        tgt = datagen.target_logits(w, z, tree.depth.cpu(), tree.n_nodes.cpu(), rep)
        rb = dd.RoundBuffers(
            n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B,
            kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
            drafter_logits=zd, root_token=rootd, q=q.to(device),
            k_cache=cache.k.to(device), v_cache=cache.v.to(device),
            block_table=None if cache.block_table is None else cache.block_table.to(device),
            prefix_len=prefix.to(device), target_logits=tgt.to(device)).allocate_outputs()
        rb.args()
        sets.append(rb)
        del cache, tgt
    torch.cuda.synchronize()
    return sets


def algorithmic_work(w, rb):
    """Algorithmic bytes / flops of each stage of one round (inputs once, no re-reads)."""
    es = 2 if w.dtype == "bf16" else 4
    nn = rb.tree.n_nodes.cpu().numpy()
    anc = rb.tree.anc.cpu().numpy().view(np.uint32)
    P = rb.prefix_len.cpu().numpy()
    acc = rb.acc.accept_len.cpu().numpy()
    popc = np.vectorize(lambda x: bin(int(x)).count("1"))
    topk_bytes = w.N * w.L * w.V * es + w.N * w.L * (w.K * 8 + 4)
    build_bytes = w.N * w.L * w.K * 8 + w.N * w.n * (5 * 4 + w.W * 4)
    kv_bytes = qo_bytes = flops = 0
    for r in range(w.N):
        vis = int(popc(anc[r, :nn[r]]).sum())
        kv_bytes += w.layers * (int(P[r]) + int(nn[r])) * w.Hkv * w.D * es * 2
        qo_bytes += w.layers * 2 * int(nn[r]) * w.Hq * w.D * es
        flops += w.layers * 4 * w.Hq * w.D * (int(nn[r]) * int(P[r]) + vis)
    accept_bytes = int(nn.sum()) * w.V * es + int(((acc - 1) * 2 * 2).sum()) * w.layers * w.Hkv * w.D * es
    return {
        "topk": {"bytes": topk_bytes, "flops": 0},
        "build": {"bytes": build_bytes, "flops": 0},
        "attn": {"bytes": kv_bytes + qo_bytes, "flops": flops},
        "accept": {"bytes": accept_bytes, "flops": 0},
    }


# ---------------------------------------------------------------- our arm

def stage_workspaces(w, rb):
    """Zero-filled workspaces of the separate stage calls of ``rb``, one per
    stage and apart from the round's own: each stage's counters and tickets
    live at the start of its workspace, so sharing one buffer would let one
    stage's scratch overwrite another's counters."""
    import ctypes
    import draft_tree_build_ddtree_b200 as dd
    if getattr(rb, "_stage_ws", None) is None:
        lib = dd.lib()
        dev = rb.drafter_logits.device
        sizes = {"topk": lib.ddtree_topk_workspace_bytes(w.N * w.L, w.V, w.K),
                 "attn": lib.ddtree_attn_workspace_bytes(ctypes.byref(rb.kv), w.B),
                 "accept": lib.ddtree_accept_workspace_bytes(w.N, w.B, w.V)}
        rb._stage_ws = {k: torch.zeros(max(256, int(n)), dtype=torch.uint8, device=dev) for k, n in sizes.items()}
    return rb._stage_ws


def stage_calls(w, rb):
    """The four stages of ``rb`` as separate library calls (the round's buffers,
    each stage's own workspace)."""
    import draft_tree_build_ddtree_b200 as dd
    ids = rb.ids.reshape(-1, w.K)
    lp = rb.lp.reshape(-1, w.K)
    ws = stage_workspaces(w, rb)

    def topk():
        dd.ddtree_topk(rb.drafter_logits.reshape(-1, w.V), w.K, ids=ids, lp=lp, lse=rb.lse, ws=ws["topk"])

    def build():
        dd.ddtree_build(rb.ids, rb.lp, rb.root_token, w.B, out=rb.tree)

    def attn():
        dd.ddtree_tree_attn(rb.q, rb.k_cache, rb.v_cache, rb.kv, rb.prefix_len, rb.tree.anc, rb.tree.n_nodes, w.B,
                            block_table=rb.block_table, out=rb.attn_out, out_lse=rb.attn_lse, ws=ws["attn"])

    def accept():
        dd.ddtree_accept(rb.target_logits, rb.tree.node_token, rb.tree.parent, rb.tree.n_nodes, w.L, rb.prefix_len,
                         rb.k_cache, rb.v_cache, rb.kv, rb.block_table, out=rb.acc, ws=ws["accept"])

    return {"topk": topk, "build": build, "attn": attn, "accept": accept}


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream, capture_error_mode="relaxed"):
        fn()
    return g


def run_ours(a):
    import draft_tree_build_ddtree_b200 as dd
    rank, world, local = dist_env()
    init_dist(world)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = workload_from_args(a)
    per_set = set_bytes(w)
    R = max(2, math.ceil(2 * L2_BYTES / per_set) + 1)
    sets = make_sets(w, R, device)
    stream = torch.cuda.current_stream(device)
    use_graph = not a.no_graph

    # one warm eager round per set (one-time library set-up happens outside capture)
    for rb in sets:
        dd.ddtree_round(rb, rb._args)
    torch.cuda.synchronize()
    if use_graph:
        side = torch.cuda.Stream(device)
        graphs = [capture(lambda rb=rb: dd.ddtree_round(rb, rb._args), side) for rb in sets]
        step = [g.replay for g in graphs]
    else:
        step = [lambda rb=rb: dd.ddtree_round(rb, rb._args) for rb in sets]

    for i in range(R):                   # every graph once: its upload happens before any timing
        step[i]()
    torch.cuda.synchronize()

    for i in range(a.warmup):
        step[i % R]()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    # ---- the timed region: exactly K steps ----
    barrier(device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(a.steps):
        step[i % R]()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(device)
    clocks.stop()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, device)
    value = aggregate_rate(a.steps, world, ms_max / 1e3)
    status = dd.device_status()

    # ---- per-stage kernel times, with cold caches as in the rounds: a graph of
    #      (L2 flush, stage on set k) for every set, minus the same graph of
    #      flushes alone ----
    names = ("topk", "build", "attn", "accept")
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def timed(fn, n):
        if use_graph:
            g = capture(fn, side)
            run = g.replay
        else:
            run = fn
        run()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            run()
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    reps = max(3, min(20, a.steps // R))
    t_flush = timed(lambda: [flush_buf.zero_() for _ in range(R)], reps)
    stage_ms = {}
    for name in names:
        fns = [stage_calls(w, rb)[name] for rb in sets]

        def flushed(fns=fns):
            for f in fns:
                flush_buf.zero_()
                f()

        stage_ms[name] = max(0.0, timed(flushed, reps) - t_flush) / (reps * R)
    del flush_buf
    # restore the caches the stage runs compacted are irrelevant: sizes do not change

    work = algorithmic_work(w, sets[0])
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    tflops = float(peaks["bf16_tflops"])
    ridge = tflops * 1e12 / (hbm * 1e9)
    stages = {}
    for name, t in stage_ms.items():
        wk = work[name]
        d = {"us": t * 1e3, "bytes": wk["bytes"], "flops": wk["flops"],
             "gbs": wk["bytes"] / (t * 1e-3) / 1e9}
        d["hbm_frac"] = d["gbs"] / hbm
        if wk["flops"]:
            d["tflops"] = wk["flops"] / (t * 1e-3) / 1e12
            d["tensor_frac"] = d["tflops"] / tflops
            d["intensity"] = wk["flops"] / wk["bytes"]
        stages[name] = d
    dom = max((n for n in stages if n != "build"), key=lambda n: stages[n]["us"])
    ds = stages[dom]
    if dom == "attn" and ds["intensity"] > ridge:
        roof = {"bound": "tensor", "achieved": ds["tflops"], "peak": tflops, "unit": "TFLOP/s",
                "frac": ds["tflops"] / tflops}
    else:
        roof = {"bound": "hbm", "achieved": ds["gbs"], "peak": hbm, "unit": "GB/s", "frac": ds["gbs"] / hbm}
    roof.update({"kernel": dom, "traffic": measured_traffic(w.name, dom), "peak_source": f"{peak_kind} (MEASURED_PEAKS.json burst)"
                 if peak_kind == "measured" else "fallback"})

    # ---- end to end through the host-buffer API ----
    e2e = None
    if not a.no_e2e:
        from draft_tree_build_ddtree_b200 import host_api
        hosts = [host_api.make_host_round(rb) for rb in sets]
        k_e2e = max(3, min(a.steps, 200))
        for i in range(2):
            host_api.round_from_host(sets[i % R], hosts[i % R], sets[i % R]._args)
        torch.cuda.synchronize()
        barrier(device)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for i in range(k_e2e):
            host_api.round_from_host(sets[i % R], hosts[i % R], sets[i % R]._args)
        f1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(f0.elapsed_time(f1), device)
        e2e = {"value": aggregate_rate(k_e2e, world, e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": hosts[0].h2d_bytes, "d2h_bytes_per_step": hosts[0].d2h_bytes,
               "steps": k_e2e}

    launches_per_round = dd.ddtree_round_launch_count(sets[0], sets[0]._args)
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, budget_s=12.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms_max / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": workload_label(w),
                       "config_id": w.cfg, "n_req": w.N, "parallelism": f"replicas x{world}",
                       "l2": f"{R} rotating input sets of {per_set / 1e6:.1f} MB (> 2x L2)",
                       "launch": "cuda graph per round" if use_graph else "eager"},
            "stages_us": {k: round(v["us"], 3) for k, v in stages.items()},
            "stages": stages,
            "roofline": roof,
            "gpu_launches": launches_per_round * a.steps,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "device_status": status,
            "accept_len_mean": float(sets[0].acc.accept_len.float().mean().item()),
        }
        print(json.dumps(line))
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------- the oracle (CPU baseline / reference arm)

def oracle_round_sample(w, z, root, q, cache, prefix, tgt, frac_rows=1, node_limit=None, head_limit=None,
                        layer_limit=None):
    """Time the oracle on a sample of one round; return extrapolated seconds per round and a description."""
    import oracle
    t = {}
    rows = z.reshape(-1, w.V)
    nrows = rows.shape[0]
    take = max(1, min(nrows, frac_rows))
    t0 = time.perf_counter()
    ids, lp32, _, _ = oracle.topk(rows[:take].to(torch.float64).numpy(), w.K)
    t["topk"] = (time.perf_counter() - t0) * nrows / take
    # the heap runs on the full table of request 0 (cheap); use the sampled rows' table tiled
    full_ids = np.tile(ids, (math.ceil(w.L / take), 1))[:w.L]
    full_lp = np.sort(np.tile(lp32, (math.ceil(w.L / take), 1))[:w.L], axis=1)[:, ::-1].copy()
    t0 = time.perf_counter()
    tree = oracle.build_tree(full_ids, full_lp, int(root[0]), w.B)
    t["build"] = (time.perf_counter() - t0) * w.N
    st = oracle.stack_trees([tree])
    nodes = list(range(tree.n_nodes))[:node_limit] if node_limit else None
    heads = list(range(w.Hq))[:head_limit] if head_limit else None
    layers = list(range(w.layers))[:layer_limit] if layer_limit else None
    qq = q[:, :1].to(torch.float64).numpy()
    kk = cache.k[:, :1].to(torch.float64).numpy() if cache.block_table is None else None
    vv = cache.v[:, :1].to(torch.float64).numpy() if cache.block_table is None else None
    if kk is None:
        # paged pools: gather request 0's logical slots into a contiguous view
        tb = cache.block_table[0]
        S = int(prefix[0]) + w.n
        nb = (S + 63) // 64
        kk = cache.k[:, tb[:nb].long()].reshape(w.layers, 1, nb * 64, w.Hkv, w.D).to(torch.float64).numpy()
        vv = cache.v[:, tb[:nb].long()].reshape(w.layers, 1, nb * 64, w.Hkv, w.D).to(torch.float64).numpy()
    t0 = time.perf_counter()
    oracle.tree_attention(qq, kk, vv, prefix[:1].numpy(), st["anc"], st["n_nodes"], datagen.default_scale(w),
                          layers=layers, nodes=nodes, heads=heads)
    frac = (len(layers) if layers else w.layers) * (len(nodes) if nodes else tree.n_nodes) * \
        (len(heads) if heads else w.Hq) / (w.layers * tree.n_nodes * w.Hq)
    t["attn"] = (time.perf_counter() - t0) / frac * w.N
    # walk: target argmax on a sample of the node rows (scaled), then the walk
    # and the compaction of the accepted path over every layer
    arows = min(tree.n_nodes, frac_rows if w.cfg == 1 else 2)
    t0 = time.perf_counter()
    oracle.argmax_rows(tgt[0, :arows].to(torch.float32).numpy())
    t_arg = (time.perf_counter() - t0) * tree.n_nodes / arows
    tg = np.zeros((tree.n_nodes, 4))
    for i in range(1, tree.n_nodes):      # a target that follows the deepest branch
        tg[st["parent"][0][i], 0] = 0.0
    t0 = time.perf_counter()
    acc = oracle.accept(tg, st["node_token"][0], st["parent"][0], tree.n_nodes, w.L, int(prefix[0]))
    oracle.compact(kk, vv, 0, acc)
    t["accept"] = (t_arg + time.perf_counter() - t0) * w.N
    desc = (f"request 0 of {w.N}; top-K on {take}/{nrows} rows; full heap; attention on "
            f"{len(layers) if layers else w.layers}/{w.layers} layers x {len(nodes) if nodes else tree.n_nodes}/"
            f"{tree.n_nodes} nodes x {len(heads) if heads else w.Hq}/{w.Hq} heads; target argmax on {arows}/"
            f"{tree.n_nodes} rows; walk + compaction; "
            f"each stage scaled to the full round")
    return sum(t.values()), t, desc


def sample_limits(w):
    """Sample sizes that keep one oracle step to tens of milliseconds."""
    if w.cfg == 1:
        return dict(frac_rows=w.N * w.L)
    return dict(frac_rows=1, node_limit=2, head_limit=2, layer_limit=1)


def cpu_baseline(w, budget_s=12.0):
    from threadpoolctl import threadpool_limits
    z = datagen.drafter_logits(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q = datagen.queries(w)
    root = datagen.root_tokens(w)
    tgt = datagen.target_logits(w, z, torch.zeros(w.N, w.n, dtype=torch.int32),
                                torch.full((w.N,), w.n, dtype=torch.int32))
    lim = sample_limits(w)
    secs, n = [], 0
    with threadpool_limits(limits=1):
        t_end = time.perf_counter() + budget_s
        while n < 1 or (time.perf_counter() < t_end and n < 50):
            s, _, desc = oracle_round_sample(w, z, root, q, cache, prefix, tgt, **lim)
            secs.append(s)
            n += 1
    per_round = statistics.median(secs)
    return {"value": 1.0 / per_round, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} sampled rounds ({desc}); numpy/BLAS limited to 1 thread"}


def run_reference(a):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    w = workload_from_args(a)
    z = datagen.drafter_logits(w)
    prefix = datagen.prefix_lengths(w)
    cache = datagen.kv_cache(w, prefix)
    q = datagen.queries(w)
    root = datagen.root_tokens(w)
    tgt = datagen.target_logits(w, z, torch.zeros(w.N, w.n, dtype=torch.int32),
                                torch.full((w.N,), w.n, dtype=torch.int32))
    lim = sample_limits(w)
    with threadpool_limits(limits=1):
        for _ in range(a.warmup):
            oracle_round_sample(w, z, root, q, cache, prefix, tgt, **lim)
        secs = []
        desc = ""
        for _ in range(a.steps):
            s, _, desc = oracle_round_sample(w, z, root, q, cache, prefix, tgt, **lim)
            secs.append(s)
    total = sum(secs)
    value = a.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": total / a.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_label(w), "config_id": w.cfg, "n_req": w.N},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"each step: {desc}; numpy/BLAS limited to 1 thread"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def run_profile(a):
    """A small, untimed run for ncu: one input set, then warmup + steps eager rounds.

    Kernel launch order: per input-set setup one top-K and one build, then per
    round top-K, build, tree attention (+ combine when split), argmax, walk.
    """
    import draft_tree_build_ddtree_b200 as dd
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    w = workload_from_args(a)
    rb = make_sets(w, 1, device)[0]
    for _ in range(a.warmup + a.steps):
        dd.ddtree_round(rb, rb._args)
    torch.cuda.synchronize()
    print(json.dumps({"profile_run": w.name, "rounds": a.warmup + a.steps, "device_status": dd.device_status()}))


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    elif a.profile:
        run_profile(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
