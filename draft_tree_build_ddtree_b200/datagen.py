"""Seeded synthetic inputs for one DDTree draft-and-verify round.

This module only draws random numbers and shapes them into the workloads the
library and its checker consume.  It holds none of the method's arithmetic
(no softmax, no top-K, no heap, no attention, no walk): every value it
returns is an input.  Both the CUDA path and the CPU oracle are fed the same
host tensors from here.

Workloads (one draft-and-verify round; shapes follow the pages' own setting,
a 30B-A3B-class target with block size 16 and tree budgets 64/256, in
"Accelerating Speculative Decoding with Block Diffusion Draft Trees" as
summarised on the zhichai.net DDTree deep dive, section 9, and the autobench
Qwen3-Coder-30B-A3B DDTree page, results table):

====  =================================  ===========================================
 id   name                               shape
====  =================================  ===========================================
  1   tiny_fp32                          N=1, L=4, V=512 fp32 ~N(0,3^2); K=8, B=16;
                                         Hq=2, Hkv=1, D=64, P=128, 1 layer, fp32 QKV
  2   b64_p2k                            N=1, L=16, V=151936 bf16 ~N(0,4^2) + one
                                         +8 peak per position; K=64, B=64;
                                         Hq=32, Hkv=4, D=128, P=2048, 1 layer
  3   b256_p8k_48l                       as 2 with K=256, B=256, P=8192, 48 layers
  4   batch32_ragged_paged               32 requests of the cfg-2 recipe,
                                         P_r ~ U[1024,16384], paged KV, 64-token
                                         pages in a random pool order, 1 layer
  5   sweep_p32k                         N=1, L=16, V=151936 bf16 ~N(0,sigma^2),
                                         no peak; B in {16..1024}, K=B, P=32768
====  =================================  ===========================================

Seeds: tensor role r of config c at repetition t is drawn from
``torch.Generator('cpu').manual_seed(1_000_000*c + 1000*r + t)`` (roles are
listed in ``ROLE``).  Gaussians are drawn in fp32 and rounded to bf16 with
round-to-nearest-even where the workload is bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch

ROLE = {
    "drafter": 0,
    "peaks": 1,
    "target_noise": 2,
    "q": 3,
    "k": 4,
    "v": 5,
    "prefix": 6,
    "pages": 7,
    "root": 8,
}

PAGE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    N: int            # requests in the round
    L: int            # block length (draft positions)
    V: int            # vocabulary
    K: int            # top-K kept per position
    B: int            # node budget (non-root nodes)
    dtype: str        # "bf16" or "f32" for logits and Q/K/V
    sigma: float      # drafter logit std-dev
    peak: float       # added to one uniformly drawn token per position
    target_sigma: float
    Hq: int
    Hkv: int
    D: int
    P: int            # committed prefix (fixed); 0 when drawn per request
    P_lo: int = 0     # per-request prefix range when P == 0
    P_hi: int = 0
    layers: int = 1
    paged: bool = False

    @property
    def n(self) -> int:
        return self.B + 1

    @property
    def W(self) -> int:
        return (self.n + 31) // 32

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


def workload(cfg: int, B: Optional[int] = None, sigma: Optional[float] = None,
             **overrides) -> Workload:
    """Return the workload of config ``cfg``; config 5 takes ``B`` and ``sigma``."""
    if cfg == 1:
        w = Workload(1, "tiny_fp32", 1, 4, 512, 8, 16, "f32", 3.0, 0.0, 1.0,
                     2, 1, 64, 128)
    elif cfg == 2:
        w = Workload(2, "b64_p2k", 1, 16, 151936, 64, 64, "bf16", 4.0, 8.0, 2.0,
                     32, 4, 128, 2048)
    elif cfg == 3:
        w = Workload(3, "b256_p8k_48l", 1, 16, 151936, 256, 256, "bf16", 4.0, 8.0,
                     2.0, 32, 4, 128, 8192, layers=48)
    elif cfg == 4:
        w = Workload(4, "batch32_ragged_paged", 32, 16, 151936, 64, 64, "bf16", 4.0,
                     8.0, 2.0, 32, 4, 128, 0, P_lo=1024, P_hi=16384, paged=True)
    elif cfg == 5:
        B = 64 if B is None else B
        sigma = 4.0 if sigma is None else sigma
        w = Workload(5, f"sweep_p32k_B{B}_s{sigma:g}", 1, 16, 151936, min(B, 151936),
                     B, "bf16", float(sigma), 0.0, 2.0, 32, 4, 128, 32768)
    else:
        raise ValueError(f"unknown config {cfg}")
    if overrides:
        w = dataclasses.replace(w, **overrides)
    return w


def seed_for(cfg: int, role: str, rep: int = 0) -> int:
    return 1_000_000 * cfg + 1000 * ROLE[role] + rep


def _gen(w: Workload, role: str, rep: int) -> torch.Generator:
    g = torch.Generator("cpu")
    g.manual_seed(seed_for(w.cfg, role, rep))
    return g


def _round_to(x: torch.Tensor, w: Workload) -> torch.Tensor:
    return x.to(w.torch_dtype)


def drafter_logits(w: Workload, rep: int = 0) -> torch.Tensor:
    """[N, L, V] drafter block logits in the workload dtype (CPU)."""
    g = _gen(w, "drafter", rep)
    z = torch.randn((w.N, w.L, w.V), generator=g, dtype=torch.float32) * w.sigma
    if w.peak != 0.0:
        gp = _gen(w, "peaks", rep)
        tok = torch.randint(0, w.V, (w.N, w.L), generator=gp)
        z.scatter_add_(2, tok.unsqueeze(-1),
                       torch.full((w.N, w.L, 1), w.peak, dtype=torch.float32))
    return _round_to(z, w)


def root_tokens(w: Workload, rep: int = 0) -> torch.Tensor:
    """[N] int32 bonus tokens (tree roots); config 1 uses token 0."""
    if w.cfg == 1:
        return torch.zeros(w.N, dtype=torch.int32)
    g = _gen(w, "root", rep)
    return torch.randint(0, w.V, (w.N,), generator=g).to(torch.int32)


def prefix_lengths(w: Workload, rep: int = 0) -> torch.Tensor:
    """[N] int32 committed prefix lengths."""
    if w.P > 0:
        return torch.full((w.N,), w.P, dtype=torch.int32)
    g = _gen(w, "prefix", rep)
    return torch.randint(w.P_lo, w.P_hi + 1, (w.N,), generator=g).to(torch.int32)


def slots_needed(w: Workload, prefix: torch.Tensor) -> int:
    """Cache slots one request needs: its prefix plus the B+1 tree slots."""
    return int(prefix.max().item()) + w.n


def queries(w: Workload, rep: int = 0) -> torch.Tensor:
    """[layers, N, B+1, Hq, D] tree-node queries (already rotated)."""
    g = _gen(w, "q", rep)
    q = torch.randn((w.layers, w.N, w.n, w.Hq, w.D), generator=g, dtype=torch.float32)
    return _round_to(q, w)


@dataclasses.dataclass
class KVCache:
    k: torch.Tensor                 # contiguous [layers, N, S, Hkv, D] or paged [layers, blocks, PAGE, Hkv, D]
    v: torch.Tensor
    block_table: Optional[torch.Tensor]  # [N, max_blocks] int32 when paged
    s_max: int                      # logical slots per request

    @property
    def paged(self) -> bool:
        return self.block_table is not None


def kv_cache(w: Workload, prefix: torch.Tensor, rep: int = 0,
             extra_slots: int = 0) -> KVCache:
    """KV cache holding each request's prefix and its B+1 tree slots.

    Contiguous layout: ``[layers, N, S, Hkv, D]`` with S = max(P_r) + B + 1
    (+ ``extra_slots``) rounded up to a multiple of 64.  Paged layout: a pool
    ``[layers, blocks, 64, Hkv, D]`` where request r owns ceil(S_r/64) blocks
    whose pool indices are a seeded random permutation, listed in
    ``block_table[r]`` (padded with -1).
    """
    S = slots_needed(w, prefix) + extra_slots
    S = (S + PAGE - 1) // PAGE * PAGE
    gk, gv = _gen(w, "k", rep), _gen(w, "v", rep)
    if not w.paged:
        shape = (w.layers, w.N, S, w.Hkv, w.D)
        k = torch.randn(shape, generator=gk, dtype=torch.float32)
        v = torch.randn(shape, generator=gv, dtype=torch.float32)
        return KVCache(_round_to(k, w), _round_to(v, w), None, S)
    per_req = [(int(p) + w.n + extra_slots + PAGE - 1) // PAGE for p in prefix.tolist()]
    total = sum(per_req)
    gp = _gen(w, "pages", rep)
    perm = torch.randperm(total, generator=gp).to(torch.int32)
    max_blocks = S // PAGE
    table = torch.full((w.N, max_blocks), -1, dtype=torch.int32)
    off = 0
    for r, nb in enumerate(per_req):
        table[r, :nb] = perm[off:off + nb]
        off += nb
    shape = (w.layers, total, PAGE, w.Hkv, w.D)
    k = torch.randn(shape, generator=gk, dtype=torch.float32)
    v = torch.randn(shape, generator=gv, dtype=torch.float32)
    return KVCache(_round_to(k, w), _round_to(v, w), table, max_blocks * PAGE)


def target_logits(w: Workload, drafter: torch.Tensor, depth: torch.Tensor,
                  n_nodes: torch.Tensor, rep: int = 0) -> torch.Tensor:
    """[N, B+1, V] target-verifier logits for the tree nodes.

    The row of a node at depth d is the drafter row min(d, L-1) (0-based: the
    drafter's distribution of the token after that node) plus N(0, s^2)
    noise, rounded to the workload dtype.  ``depth`` is the tree's depth
    array ([N, B+1], -1 past ``n_nodes``); rows of absent nodes get the
    noise only.  The tree itself is an input to this generator.
    """
    g = _gen(w, "target_noise", rep)
    noise = torch.randn((w.N, w.n, w.V), generator=g, dtype=torch.float32) * w.target_sigma
    base = drafter.to(torch.float32)
    d = depth.to(torch.int64).clamp(min=0, max=w.L - 1)
    rows = torch.gather(base, 1, d.unsqueeze(-1).expand(w.N, w.n, w.V))
    live = (torch.arange(w.n).unsqueeze(0) < n_nodes.to(torch.int64).unsqueeze(1))
    rows = rows * live.unsqueeze(-1).to(torch.float32)
    return _round_to(rows + noise, w)


def sweep_budgets():
    return [16, 32, 64, 128, 256, 512, 1024]


def sweep_sigmas():
    return [1.0, 4.0, 8.0]


def describe(w: Workload) -> Dict:
    d = dataclasses.asdict(w)
    d["n"] = w.n
    return d


def nbytes_of_logits(w: Workload) -> int:
    return w.N * w.L * w.V * (2 if w.dtype == "bf16" else 4)


def default_scale(w: Workload) -> float:
    return 1.0 / math.sqrt(w.D)
