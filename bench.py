#!/usr/bin/env python
"""Benchmark one DDTree draft-and-verify round (ddtree_round) on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config C] [--impl ours|reference]

A step is one ddtree_round (top-K -> tree build -> tree attention over all
of the workload's layers -> verifier walk + KV compaction) over one batch of
synthetic inputs already resident in HBM.  Steps rotate over enough input
sets that consecutive steps never find their inputs in L2.  The default
workload is b256_p8k_48l (budget 256, 8k prefix, 48 layers: the largest
single-GPU configuration); ``per_config`` adds b64_p2k, the 32-request
paged batch and the 32k-prefix sweep at B = 64 and 256.

Multi-GPU: ``--gpus N`` without a torchrun environment re-launches itself
under ``torch.distributed.run`` with N ranks.  Batch-1 workloads run as
independent replicas (weak scaling); the batched workload (config 4) is
sharded by request (request r on rank r mod N, strong scaling) and each
round ends with an NCCL all-gather of every request's accept length, next
bonus token and new prefix length.  Times are CUDA events, max over ranks.

``--impl reference`` times the CPU oracle (the checker, plain numpy) on the
host, each step one bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import socket
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
NOMINAL_HBM_GBS = 8000.0   # the workload statement's nominal HBM bandwidth (context, not the denominator)
DEFAULT_CONFIG = 3
PER_CONFIG = ((2, {}), (4, {}), (5, {"B": 64, "sigma": 4.0}), (5, {"B": 256, "sigma": 4.0}))
SUSTAINED_AFTER_S = 1.0      # a timed region at least this long is graded against the sustained peak


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG)
    ap.add_argument("--budget", type=int, default=None, help="config 5: B")
    ap.add_argument("--sigma", type=float, default=None, help="config 5: drafter logit std-dev")
    ap.add_argument("--layers", type=int, default=None, help="override the workload's attention layers "
                    "(profiling runs on a smaller case)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-graph", action="store_true", help="launch rounds eagerly instead of CUDA graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="profiling driver: one input set, warmup + steps eager rounds, no timing")
    return ap.parse_args(argv)


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from one
# ncu capture, with a hash of the kernel's sources at capture time: the value
# is reported only while the sources are unchanged (summaries under profiles/).
CSRC = os.path.join(ROOT, "draft_tree_build_ddtree_b200", "csrc")
TRAFFIC = {
    # dram__bytes_read.sum + dram__bytes_write.sum of one launch, from the ncu
    # captures summarised in profiles/ (keyed to a digest of the kernel's sources)
    ("b64_p2k", "topk"): (5070336, ("topk.cuh", "common.cuh", "exp64_table.h"), "9afe9d45b2773877"),
    ("batch32_ragged_paged", "topk"): (161479424, ("topk.cuh", "common.cuh", "exp64_table.h"), "9afe9d45b2773877"),
    # captured at 8 of the 48 layers (168,635,904 B) and scaled by 6: each
    # layer's units read that layer's K/V and write its outputs only
    ("b256_p8k_48l", "attn"): (1011815424, ("attn_tc2.cuh", "attn_tc.cuh", "common.cuh", "exp2_poly.h"),
                               "3333612cb60ec011"),
}


def sources_digest(files) -> str:
    import hashlib
    m = hashlib.sha256()
    for f in files:
        with open(os.path.join(CSRC, f), "rb") as fh:
            m.update(fh.read())
    return m.hexdigest()[:16]


def measured_traffic(workload: str, stage: str):
    entry = TRAFFIC.get((workload, stage))
    if entry is None:
        return None
    nbytes, files, digest = entry
    try:
        return nbytes if sources_digest(files) == digest else None
    except OSError:
        return None


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
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", dist_env()[2])
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120), **kw)


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


def free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def relaunch_cmd(argv, n: int, port: int):
    """The torchrun command that runs this script on n ranks of one node."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *argv]


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

def workload_of(cfg: int, over=None):
    over = dict(over or {})
    if cfg == 5:
        return datagen.workload(5, B=over.pop("B", 64), sigma=over.pop("sigma", 4.0), **over)
    return datagen.workload(cfg, **over)


def workload_from_args(a):
    over = {}
    if a.config == 5:
        over = {"B": a.budget or 64, "sigma": a.sigma or 4.0}
    if a.layers:
        over["layers"] = a.layers
    return workload_of(a.config, over)


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


def host_inputs(w, rep, device, shard=None):
    """One input set on the host: drafter logits, prefix, cache, queries,
    roots and the target logits (which follow the tree the library builds
    from the drafter logits).  ``shard``: the request indices to keep."""
    import draft_tree_build_ddtree_b200 as dd
    z = datagen.drafter_logits(w, rep)
    prefix = datagen.prefix_lengths(w, rep)
    cache = datagen.kv_cache(w, prefix, rep)
    q = datagen.queries(w, rep)
    root = datagen.root_tokens(w, rep)
    ids, lp, _ = dd.ddtree_topk(z.to(device).reshape(-1, w.V), w.K)
    tree = dd.ddtree_build(ids.reshape(w.N, w.L, w.K), lp.reshape(w.N, w.L, w.K), root.to(device), w.B)
    tgt = datagen.target_logits(w, z, tree.depth.cpu(), tree.n_nodes.cpu(), rep)
    if shard is not None:
        idx = torch.tensor(shard, dtype=torch.long)
        z, prefix, root, tgt, q = z[idx], prefix[idx], root[idx], tgt[idx], q[:, idx]
        if cache.block_table is None:
            cache = datagen.KVCache(cache.k[:, idx].contiguous(), cache.v[:, idx].contiguous(), None, cache.s_max)
        else:
            cache = datagen.KVCache(cache.k, cache.v, cache.block_table[idx].contiguous(), cache.s_max)
    return dict(z=z, prefix=prefix, cache=cache, q=q.contiguous(), root=root, tgt=tgt.contiguous())


def to_round(w, h, device):
    import draft_tree_build_ddtree_b200 as dd
    cache = h["cache"]
    rb = dd.RoundBuffers(
        n_req=w.N, L=w.L, V=w.V, K=w.K, B=w.B,
        kv=dd.kv_desc_for(cache.k, w.N, w.Hq, cache.block_table),
        drafter_logits=h["z"].to(device), root_token=h["root"].to(device), q=h["q"].to(device),
        k_cache=cache.k.to(device), v_cache=cache.v.to(device),
        block_table=None if cache.block_table is None else cache.block_table.to(device),
        prefix_len=h["prefix"].to(device), target_logits=h["tgt"].to(device)).allocate_outputs()
    rb.args()
    return rb


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


def stage_report(w, work, stage_ms, peaks, long_region: bool):
    """Per-stage µs, achieved bandwidth / flop rate and roof fractions."""
    hbm = float(peaks["hbm_gbs"])
    burst = float(peaks["bf16_tflops"])
    sust = float(peaks.get("bf16_tflops_sustained", burst))
    tensor_peak = sust if long_region else burst
    ridge = tensor_peak * 1e12 / (hbm * 1e9)
    stages = {}
    for name, t in stage_ms.items():
        wk = work[name]
        d = {"us": t * 1e3, "bytes": wk["bytes"], "flops": wk["flops"], "gbs": wk["bytes"] / (t * 1e-3) / 1e9}
        d["hbm_frac"] = d["gbs"] / hbm
        d["hbm_frac_nominal"] = d["gbs"] / NOMINAL_HBM_GBS
        if wk["flops"]:
            d["tflops"] = wk["flops"] / (t * 1e-3) / 1e12
            d["tensor_frac_burst"] = d["tflops"] / burst
            d["tensor_frac_sustained"] = d["tflops"] / sust
            d["intensity"] = wk["flops"] / wk["bytes"]
            d["bound"] = "tensor" if d["intensity"] > ridge else "hbm"
        else:
            d["bound"] = "hbm" if name != "build" else "latency"
        d["frac"] = (d["tflops"] / tensor_peak) if d["bound"] == "tensor" else d["hbm_frac"]
        stages[name] = d
    return stages, tensor_peak


def measure(w, a, device, steps, warmup, shard=None, world=1, rank=0, clocks=None, gather=False, keep_host=False):
    """Build the input sets of ``w`` (this rank's ``shard`` of requests),
    time ``steps`` rounds and each stage; returns a result dict."""
    import draft_tree_build_ddtree_b200 as dd
    from draft_tree_build_ddtree_b200 import serving
    w_run = w if shard is None else dataclasses.replace(w, N=len(shard))
    per_set = set_bytes(w_run)
    R = max(2, math.ceil(2 * L2_BYTES / per_set) + 1)
    hosts = [host_inputs(w, rep, device, shard) for rep in range(R)]
    sets = [to_round(w_run, h, device) for h in hosts]
    host0 = hosts[0] if keep_host else None
    del hosts
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    use_graph = not a.no_graph
    for rb in sets:                     # one eager round per set: one-time set-up outside any capture
        dd.ddtree_round(rb, rb._args)
    torch.cuda.synchronize()
    side = torch.cuda.Stream(device)
    if use_graph:
        graphs = [capture(lambda rb=rb: dd.ddtree_round(rb, rb._args), side) for rb in sets]
        rounds = [g.replay for g in graphs]
    else:
        rounds = [lambda rb=rb: dd.ddtree_round(rb, rb._args) for rb in sets]

    def step(i):
        rounds[i % R]()
        if gather:                      # the batch's per-request outcome, in request order, on every rank
            rb = sets[i % R]
            local = torch.stack([rb.acc.accept_len, rb.acc.next_bonus, rb.acc.new_prefix_len], dim=1)
            serving.gather_by_request(local, w.N, world, rank)

    for i in range(R):                  # every graph once: its upload happens before any timing
        step(i)
    torch.cuda.synchronize()
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
        time.sleep(0.3)
    barrier(device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(device)
    if clocks is not None:
        clocks.stop()
    ms = e0.elapsed_time(e1)
    ms_max = max_over_ranks(ms, device)
    status = dd.device_status()

    # the spread of single rounds (each bracketed by its own events), and
    # rounds launched eagerly instead of from CUDA graphs
    n_each = min(steps, 200)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_each)]
    for i, (a0, a1) in enumerate(evs):
        a0.record(stream)
        step(i)
        a1.record(stream)
    torch.cuda.synchronize()
    each_us = sorted(a0.elapsed_time(a1) * 1e3 for a0, a1 in evs)
    pct = lambda q: each_us[min(len(each_us) - 1, int(round(q * (len(each_us) - 1))))]
    round_us = {"p10": round(pct(0.1), 3), "median": round(pct(0.5), 3), "p90": round(pct(0.9), 3),
                "rounds": n_each}
    eager_rps = None
    if use_graph and not gather:
        n_eager = min(steps, 50)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(n_eager):
            rb = sets[i % R]
            dd.ddtree_round(rb, rb._args)
        t1.record(stream)
        torch.cuda.synchronize()
        eager_rps = n_eager / (t0.elapsed_time(t1) / 1e3)

    # per-stage times with cold caches as in the rounds: a graph of (L2 flush,
    # stage on set k) for every set, minus the same graph of flushes alone
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def timed(fn, n):
        run = capture(fn, side).replay if use_graph else fn
        run()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(n):
            run()
        t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    reps = max(3, min(20, steps // R))
    t_flush = timed(lambda: [flush_buf.zero_() for _ in range(R)], reps)
    work = algorithmic_work(w_run, sets[0])
    stage_ms = {}
    stage_l2 = {}
    for name in ("topk", "build", "attn", "accept"):
        fns = [stage_calls(w_run, rb)[name] for rb in sets]
        if work[name]["bytes"] > L2_BYTES:
            # one launch reads more than the L2 holds: the sets in rotation
            # reach it cold without a flush (whose dirty lines would be
            # written back during the stage)
            def plain(fns=fns):
                for f in fns:
                    f()
            stage_ms[name] = timed(plain, reps) / (reps * R)
            stage_l2[name] = "inputs larger than L2"
            continue

        def flushed(fns=fns):
            for f in fns:
                flush_buf.zero_()
                f()

        stage_ms[name] = max(1e-6, timed(flushed, reps) - t_flush) / (reps * R)
        stage_l2[name] = "L2 flushed before each launch"
    del flush_buf
    return dict(w=w_run, sets=sets, R=R, per_set=per_set, ms=ms_max, steps=steps, status=status,
                stage_ms=stage_ms, stage_l2=stage_l2, work=work, round_us=round_us, eager_rps=eager_rps,
                use_graph=use_graph, host0=host0,
                launches=dd.ddtree_round_launch_count(sets[0], sets[0]._args),
                accept_len_mean=float(torch.cat([rb.acc.accept_len.float() for rb in sets]).mean().item()))


def run_ours(a):
    import draft_tree_build_ddtree_b200 as dd
    from draft_tree_build_ddtree_b200 import serving
    rank, world, local = dist_env()
    if world != a.gpus:
        raise SystemExit(f"bench.py: --gpus {a.gpus} but WORLD_SIZE is {world}")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world)
    w = workload_from_args(a)
    sharded = w.N > 1 and world > 1          # the batched workload splits by request
    shard = serving.shard_of(w.N, world, rank) if sharded else None
    clocks = ClockSampler(local)
    m = measure(w, a, device, a.steps, a.warmup, shard=shard, world=world, rank=rank, clocks=clocks,
                gather=sharded, keep_host=(rank == 0 and world == 1 and not a.no_cpu_baseline))
    if sharded:
        value = a.steps / (m["ms"] / 1e3)    # whole-batch rounds per second
    else:
        value = aggregate_rate(a.steps, world, m["ms"] / 1e3)
    peaks, peak_kind = load_peaks()
    long_region = m["ms"] / 1e3 >= SUSTAINED_AFTER_S
    stages, tensor_peak = stage_report(m["w"], m["work"], m["stage_ms"], peaks, long_region)
    dom = max((n for n in stages if n != "build"), key=lambda n: stages[n]["us"])
    ds = stages[dom]
    if ds["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": ds["tflops"], "peak": tensor_peak, "unit": "TFLOP/s",
                "frac": ds["tflops"] / tensor_peak}
    else:
        roof = {"bound": "hbm", "achieved": ds["gbs"], "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                "frac": ds["gbs"] / float(peaks["hbm_gbs"])}
    roof.update({"kernel": dom, "traffic": measured_traffic(w.name, dom),
                 "peak_source": (f"of {peak_kind} (MEASURED_PEAKS.json "
                                 f"{'sustained' if long_region and ds['bound'] == 'tensor' else 'burst'})")})

    # ---- end to end through the C ABI's host-buffer round ----
    e2e = None
    if not a.no_e2e:
        from draft_tree_build_ddtree_b200 import host_api
        sets, R = m["sets"], m["R"]
        hosts = [host_api.make_host_round(rb, rb._args) for rb in sets]
        k_e2e = max(3, min(a.steps, 100))
        stream = torch.cuda.current_stream(device)
        # one stream per input set (each set owns its device buffers and
        # workspace): consecutive rounds overlap one round's copies with the
        # other's kernels.  The request-sharded path keeps one stream, so that
        # every rank issues its collectives in one order on one stream.
        streams = [stream] if sharded else [torch.cuda.Stream(device) for _ in range(R)]
        for i in range(R):
            host_api.round_from_host(sets[i], hosts[i], sets[i]._args)
        torch.cuda.synchronize()
        barrier(device)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for st in streams:
            st.wait_event(f0)
        for i in range(k_e2e):
            with torch.cuda.stream(streams[i % len(streams)]):
                host_api.round_from_host(sets[i % R], hosts[i % R], sets[i % R]._args)
            if sharded:
                rb = sets[i % R]
                serving.gather_by_request(torch.stack([rb.acc.accept_len, rb.acc.next_bonus,
                                                       rb.acc.new_prefix_len], dim=1), w.N, world, rank)
        for st in streams:
            stream.wait_event(st.record_event())
        f1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(f0.elapsed_time(f1), device)
        e_val = k_e2e / (e_ms / 1e3) if sharded else aggregate_rate(k_e2e, world, e_ms / 1e3)
        e2e = {"value": e_val, "unit": UNIT, "h2d_bytes_per_step": hosts[0].h2d_bytes,
               "d2h_bytes_per_step": hosts[0].d2h_bytes, "steps": k_e2e, "streams": len(streams),
               "api": "ddtree_round_host (C ABI): pinned host inputs, round, host results"}
        del hosts

    per_config = None
    if world == 1 and not a.no_per_config:
        per_config = {}
        for cfg, over in PER_CONFIG:
            wc = workload_of(cfg, over)
            if wc.name == w.name:
                continue
            mc = measure(wc, a, device, max(50, min(a.steps, 500)), max(3, a.warmup))
            long_c = mc["ms"] / 1e3 >= SUSTAINED_AFTER_S
            st_c, _ = stage_report(mc["w"], mc["work"], mc["stage_ms"], peaks, long_c)
            per_config[wc.name] = {
                "workload": workload_label(wc), "rounds_per_s": mc["steps"] / (mc["ms"] / 1e3),
                "ms_per_round": mc["ms"] / mc["steps"], "steps": mc["steps"], "device_status": mc["status"],
                "stages_us": {k: round(v["us"], 3) for k, v in st_c.items()},
                "stages_l2": mc["stage_l2"],
                "roof": {k: {kk: v[kk] for kk in ("bound", "frac", "hbm_frac", "hbm_frac_nominal", "tensor_frac_burst",
                                                  "tensor_frac_sustained", "gbs", "tflops") if kk in v}
                         for k, v in st_c.items()},
                "accept_len_mean": mc["accept_len_mean"]}
            del mc
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        cpu = cpu_baseline(w, m["host0"], budget_s=15.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": m["ms"] / a.steps, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": workload_label(w), "config_id": w.cfg, "n_req": w.N,
                       "parallelism": (f"requests sharded over {world} ranks (r mod {world})" if sharded
                                       else f"replicas x{world}"),
                       "l2": f"{m['R']} rotating input sets of {m['per_set'] / 1e6:.1f} MB (> 2x L2)",
                       "launch": "cuda graph per round" if m["use_graph"] else "eager"},
            "round_us": m["round_us"],
            "eager_rounds_per_s": m["eager_rps"],
            "stages_us": {k: round(v["us"], 3) for k, v in stages.items()},
            "stages_l2": m["stage_l2"],
            "stages": stages,
            "roofline": roof,
            "gpu_launches": m["launches"] * a.steps,
            "clocks": clocks.summary(),
            "e2e": e2e,
            "cpu_baseline": cpu,
            "per_config": per_config,
            "device_status": m["status"],
            "accept_len_mean": m["accept_len_mean"],
        }
        print(json.dumps(line))
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


# ---------------------------------------------------------------- the oracle (CPU baseline / reference arm)

def oracle_sample(w):
    """The part of one round the oracle runs in a timed step, and the factor
    that scales each stage's time to the full round.  The dense attention is
    the slow part (8 ms per node and head at P = 8192): configs 1 and 2 run
    in full, the larger ones on a stated subset."""
    if w.cfg in (1, 2):
        return dict(reqs=list(range(w.N)), layers=None, heads=None)
    if w.cfg == 4:
        return dict(reqs=[0, 1, 2, 3], layers=None, heads=[0, 16])
    return dict(reqs=[0], layers=[0], heads=[0])


def oracle_round(w, h, sample):
    """The oracle on one round's real inputs (``h``: the host copy of an
    input set): top-K of the sampled requests' rows, their heaps, dense
    attention on the sampled layers and heads (every node), the target
    argmax of every live node, the walk, and the compaction of every layer.
    Returns (seconds scaled to the full round, per-stage seconds, description)."""
    import oracle
    reqs = sample["reqs"]
    n_r = len(reqs)
    idx = torch.tensor(reqs, dtype=torch.long)
    z = h["z"][idx].to(torch.float64).numpy()
    t = {}
    t0 = time.perf_counter()
    ids, lp32, _, _ = oracle.topk(z, w.K)
    t["topk"] = time.perf_counter() - t0
    root = h["root"][idx].numpy()
    t0 = time.perf_counter()
    trees = oracle.build_trees(ids, lp32, root, w.B)
    t["build"] = time.perf_counter() - t0
    st = oracle.stack_trees(trees)
    prefix = h["prefix"][idx].numpy()
    cache = h["cache"]
    layers = list(range(w.layers)) if sample["layers"] is None else sample["layers"]
    t["attn"] = 0.0
    for l in layers:
        if cache.block_table is None:
            kk = cache.k[l:l + 1, idx].to(torch.float64).numpy()
            vv = cache.v[l:l + 1, idx].to(torch.float64).numpy()
        else:       # the sampled requests' pages gathered into contiguous rows
            S = int(prefix.max()) + w.n
            nb = (S + 63) // 64
            tb = cache.block_table[idx, :nb].clamp(min=0).long()
            kk = cache.k[l][tb].reshape(1, n_r, nb * 64, w.Hkv, w.D).to(torch.float64).numpy()
            vv = cache.v[l][tb].reshape(1, n_r, nb * 64, w.Hkv, w.D).to(torch.float64).numpy()
        qq = h["q"][l:l + 1, idx].to(torch.float64).numpy()
        t0 = time.perf_counter()
        oracle.tree_attention(qq, kk, vv, prefix, st["anc"], st["n_nodes"], datagen.default_scale(w),
                              heads=sample["heads"])
        t["attn"] += time.perf_counter() - t0
    tgt = h["tgt"][idx].to(torch.float32).numpy()
    kb = cache.k.view(torch.int16).numpy() if w.dtype == "bf16" else cache.k.numpy()
    vb = cache.v.view(torch.int16).numpy() if w.dtype == "bf16" else cache.v.numpy()
    table = None if cache.block_table is None else cache.block_table.numpy()
    t0 = time.perf_counter()
    for j, r in enumerate(reqs):
        acc = oracle.accept(tgt[j], st["node_token"][j], st["parent"][j], int(st["n_nodes"][j]), w.L, int(prefix[j]))
        oracle.compact(kb, vb, r, acc, block_table=table)
    t["accept"] = time.perf_counter() - t0
    heads = w.Hq if sample["heads"] is None else len(sample["heads"])
    f_req = w.N / n_r
    f_attn = f_req * (w.layers / len(layers)) * (w.Hq / heads)
    full = (t["topk"] + t["build"] + t["accept"]) * f_req + t["attn"] * f_attn
    desc = (f"real inputs of one round; requests {n_r}/{w.N}: top-K of all their rows, full heap, target argmax of "
            f"every live node, walk, compaction of all {w.layers} layers; dense attention on "
            f"{len(layers)}/{w.layers} layers x {heads}/{w.Hq} query heads x every node"
            + ("" if f_attn == 1.0 else f"; attention time x{f_attn:g} and the rest x{f_req:g} to the full round"))
    return full, t, desc


def cpu_baseline(w, h, budget_s=15.0):
    from threadpoolctl import threadpool_limits
    sample = oracle_sample(w)
    secs, n, desc = [], 0, ""
    with threadpool_limits(limits=1):
        t_end = time.perf_counter() + budget_s
        while n < 1 or (time.perf_counter() < t_end and n < 20):
            s, _, desc = oracle_round(w, h, sample)
            secs.append(s)
            n += 1
    per_round = statistics.median(secs)
    out = {"value": 1.0 / per_round, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{n} timed oracle rounds ({desc}); numpy/BLAS limited to 1 thread"}
    # the same sample with numpy's BLAS on every host core (its dense
    # attention products are the part that runs in parallel)
    cores = os.cpu_count() or 1
    if cores > 1:
        secs_all = []
        with threadpool_limits(limits=cores):
            t_end = time.perf_counter() + budget_s / 2
            while not secs_all or (time.perf_counter() < t_end and len(secs_all) < 10):
                s, _, _ = oracle_round(w, h, sample)
                secs_all.append(s)
        out["all_cores"] = {"value": 1.0 / statistics.median(secs_all), "cores": cores,
                            "sample": f"{len(secs_all)} timed oracle rounds, numpy/BLAS on {cores} threads"}
    return out


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
    # the target rows follow the oracle's own tree on this host (no GPU here)
    import oracle
    ids, lp32, _, _ = oracle.topk(z.to(torch.float64).numpy(), w.K)
    st = oracle.stack_trees(oracle.build_trees(ids, lp32, root.numpy(), w.B))
    tgt = datagen.target_logits(w, z, torch.from_numpy(st["depth"]), torch.from_numpy(st["n_nodes"]))
    h = dict(z=z, prefix=prefix, cache=cache, q=q, root=root, tgt=tgt)
    sample = oracle_sample(w)
    desc = ""
    with threadpool_limits(limits=1):
        for _ in range(a.warmup):
            oracle_round(w, h, sample)
        step_s, full_s = [], []
        for _ in range(a.steps):
            t0 = time.perf_counter()
            full, _, desc = oracle_round(w, h, sample)
            step_s.append(time.perf_counter() - t0)
            full_s.append(full)
    total = sum(step_s)
    value = a.steps / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": total / a.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_label(w), "config_id": w.cfg, "n_req": w.N},
            "step": f"one oracle round on the stated sample: {desc}",
            "extrapolated_full_round": {"rounds_per_s": a.steps / sum(full_s),
                                        "ms_per_round": sum(full_s) / a.steps * 1e3,
                                        "method": "each stage's sampled time scaled by its sample fraction"},
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
    rb = to_round(w, host_inputs(w, 0, device), device)
    for _ in range(a.warmup + a.steps):
        dd.ddtree_round(rb, rb._args)
    torch.cuda.synchronize()
    print(json.dumps({"profile_run": w.name, "rounds": a.warmup + a.steps, "device_status": dd.device_status()}))


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    a = parse(argv)
    if a.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(subprocess.call(relaunch_cmd(argv, a.gpus, free_port())))
    if a.impl == "reference":
        run_reference(a)
    elif a.profile:
        run_profile(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
