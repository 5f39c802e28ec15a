"""Host-buffer round: pinned host inputs in, host results out, through the C ABI.

``round_from_host`` is the call a user without device-resident logits makes:
one ``ddtree_round_host`` call copies the round's inputs from pinned host
memory into the device buffers (drafter logits, root tokens, tree-node
queries, target logits, prefix lengths and, for contiguous caches, the tree
nodes' K/V rows into the cache tail), runs the round and copies its results
back, all on the current stream.  This module only marshals the pointers.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Dict

import torch

from . import RoundArgs, RoundBuffers, _check, _stream, lib

_vp = ctypes.c_void_p

IO_FIELDS = ("drafter_logits", "root_token", "q", "target_logits", "prefix_len", "tree_k", "tree_v",
             "attn_out", "node_token", "parent", "n_nodes", "path", "accept_len", "next_bonus", "new_prefix_len")


class RoundHostIO(ctypes.Structure):
    _fields_ = [(f, _vp) for f in IO_FIELDS]


INPUT_FIELDS = ("drafter_logits", "root_token", "q", "target_logits", "prefix_len")
TREE_OUTPUTS = ("node_token", "parent", "n_nodes")
ACCEPT_OUTPUTS = ("path", "accept_len", "next_bonus", "new_prefix_len")


@dataclasses.dataclass
class HostRound:
    """Pinned host mirrors of one round's per-step inputs and results."""
    inputs: Dict[str, torch.Tensor]
    outputs: Dict[str, torch.Tensor]
    io: RoundHostIO
    h2d_bytes: int = 0
    d2h_bytes: int = 0


def tree_tail(rb: RoundBuffers, cache: torch.Tensor) -> torch.Tensor:
    """[layers, n_req, B+1, Hkv, D]: the rows at slots P_r .. P_r + B (contiguous caches)."""
    P = rb.prefix_len.cpu().tolist()
    return torch.stack([cache[:, r, P[r]:P[r] + rb.B + 1] for r in range(rb.n_req)], dim=1)


def make_host_round(rb: RoundBuffers, args: RoundArgs = None) -> HostRound:
    """Pinned host buffers holding ``rb``'s per-step inputs and room for its results."""
    ins = {f: getattr(rb, f).to("cpu").pin_memory() for f in INPUT_FIELDS}
    if rb.block_table is None:
        ins["tree_k"] = tree_tail(rb, rb.k_cache).to("cpu").contiguous().pin_memory()
        ins["tree_v"] = tree_tail(rb, rb.v_cache).to("cpu").contiguous().pin_memory()
    outs = {"attn_out": torch.empty_like(rb.attn_out, device="cpu").pin_memory()}
    for f in TREE_OUTPUTS:
        outs[f] = torch.empty_like(getattr(rb.tree, f), device="cpu").pin_memory()
    for f in ACCEPT_OUTPUTS:
        outs[f] = torch.empty_like(getattr(rb.acc, f), device="cpu").pin_memory()
    io = RoundHostIO()
    for f in IO_FIELDS:
        t = ins.get(f, outs.get(f))
        setattr(io, f, None if t is None else t.data_ptr())
    a = rb.args() if args is None else args
    h2d, d2h = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    if lib().ddtree_round_host_bytes(ctypes.byref(a), ctypes.byref(io), ctypes.byref(h2d), ctypes.byref(d2h)) != 0:
        raise ValueError("invalid host round")
    return HostRound(ins, outs, io, int(h2d.value), int(d2h.value))


def round_from_host(rb: RoundBuffers, host: HostRound, args: RoundArgs = None) -> HostRound:
    """H2D copies of the step's inputs, one round, D2H copies of its results (one C call)."""
    a = rb.args() if args is None else args
    _check(lib().ddtree_round_host(ctypes.byref(a), ctypes.byref(host.io), _stream()), "ddtree_round_host")
    return host
