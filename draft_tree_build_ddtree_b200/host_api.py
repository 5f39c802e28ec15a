"""Host-buffer entry point of the round: pinned host inputs in, host results out.

``round_from_host`` is the call a user without device-resident logits makes:
it copies one round's inputs from pinned host memory into the device
buffers, runs ``ddtree_round`` and copies the round's results back, all on
the current stream.  Copies are torch's (plumbing); the round itself is the
library's.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List

import torch

from . import RoundBuffers, ddtree_round


@dataclasses.dataclass
class HostRound:
    """Pinned host mirrors of one round's per-step inputs and results."""
    inputs: Dict[str, torch.Tensor]
    outputs: Dict[str, torch.Tensor]
    tail_views: List[torch.Tensor]   # device views the tree K/V rows are copied into

    @property
    def h2d_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.inputs.values())

    @property
    def d2h_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in self.outputs.values())


INPUT_FIELDS = ("drafter_logits", "root_token", "q", "target_logits", "prefix_len")
OUTPUT_FIELDS = ("attn_out",)
TREE_OUTPUTS = ("node_token", "parent", "n_nodes")
ACCEPT_OUTPUTS = ("path", "accept_len", "next_bonus", "new_prefix_len")


def tree_tail_slots(rb: RoundBuffers) -> List[torch.Tensor]:
    """Device views of each request's B+1 tree slots (contiguous caches only)."""
    views = []
    P = rb.prefix_len.cpu().tolist()
    for cache in (rb.k_cache, rb.v_cache):
        for r in range(rb.n_req):
            views.append(cache[:, r, P[r]:P[r] + rb.B + 1])
    return views


def make_host_round(rb: RoundBuffers) -> HostRound:
    """Pinned host buffers shaped like ``rb``'s per-step inputs and results."""
    ins = {f: torch.empty_like(getattr(rb, f), device="cpu").pin_memory() for f in INPUT_FIELDS}
    for f in INPUT_FIELDS:
        ins[f].copy_(getattr(rb, f))
    views = tree_tail_slots(rb) if rb.block_table is None else []
    for i, v in enumerate(views):
        ins[f"tree_kv_{i}"] = v.to("cpu").pin_memory()
    outs = {"attn_out": torch.empty_like(rb.attn_out, device="cpu").pin_memory()}
    for f in TREE_OUTPUTS:
        outs[f] = torch.empty_like(getattr(rb.tree, f), device="cpu").pin_memory()
    for f in ACCEPT_OUTPUTS:
        outs[f] = torch.empty_like(getattr(rb.acc, f), device="cpu").pin_memory()
    return HostRound(ins, outs, views)


def round_from_host(rb: RoundBuffers, host: HostRound, args=None) -> HostRound:
    """H2D copy of the step's inputs, one round, D2H copy of its results."""
    for f in INPUT_FIELDS:
        getattr(rb, f).copy_(host.inputs[f], non_blocking=True)
    for i, v in enumerate(host.tail_views):
        v.copy_(host.inputs[f"tree_kv_{i}"], non_blocking=True)
    ddtree_round(rb, args)
    host.outputs["attn_out"].copy_(rb.attn_out, non_blocking=True)
    for f in TREE_OUTPUTS:
        host.outputs[f].copy_(getattr(rb.tree, f), non_blocking=True)
    for f in ACCEPT_OUTPUTS:
        host.outputs[f].copy_(getattr(rb.acc, f), non_blocking=True)
    return host
