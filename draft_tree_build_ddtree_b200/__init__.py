"""Python binding of libddtree.so: one DDTree draft-and-verify round on sm_100a.

Argument marshalling only.  Every step of the round runs in the library's
CUDA kernels; PyTorch supplies device memory and the current stream.  There
is no CPU fallback: if the shared library is missing or the device is not a
CUDA device, the calls raise.

Entry points mirror the C ABI in include/ddtree.h:

    ddtree_topk(logits[rows, V], K)            -> ids, lp, lse
    ddtree_build(ids, lp, root_token, B)       -> Tree arrays
    ddtree_tree_attn(q, kv, prefix_len, tree)  -> out, lse
    ddtree_accept(target, tree, prefix_len...) -> Accept arrays (+ in-place KV compaction)
    ddtree_round(RoundBuffers)                 -> all of the above in one call
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

import torch

__all__ = [
    "DDTreeError", "KVDesc", "lib", "ddtree_topk", "ddtree_build", "ddtree_tree_attn",
    "ddtree_accept", "ddtree_round", "device_status", "RoundBuffers", "Workspace", "Sampling",
    "ddtree_tree_kv_write", "ddtree_lmhead_argmax", "ddtree_walk",
    "BF16", "F32",
]

BF16, F32 = 0, 1
STATUS_NONFINITE, STATUS_TIMEOUT, STATUS_CAPACITY, STATUS_SETUP, STATUS_BOUNDS = 1, 2, 4, 8, 16
# DDTREE_LIBRARY=debug selects the bounds-checked build libddtree_debug.so
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libddtree_debug.so" if os.environ.get("DDTREE_LIBRARY") == "debug" else "libddtree.so")
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_ll = ctypes.c_longlong
_sz = ctypes.c_size_t


class DDTreeError(RuntimeError):
    pass


class KVDesc(ctypes.Structure):
    _fields_ = [("layers", _i), ("n_req", _i), ("Hq", _i), ("Hkv", _i), ("D", _i),
                ("scale", ctypes.c_float), ("paged", _i), ("s_max", _i),
                ("num_blocks", _i), ("max_blocks", _i)]


class Sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_double), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_ulonglong)]


class RoundArgs(ctypes.Structure):
    _fields_ = [("n_req", _i), ("L", _i), ("V", _i), ("K", _i), ("B", _i), ("dtype", _i),
                ("kv", KVDesc),
                ("drafter_logits", _vp), ("drafter_stride", _ll), ("root_token", _vp),
                ("q", _vp), ("k_cache", _vp), ("v_cache", _vp), ("block_table", _vp),
                ("prefix_len", _vp), ("target_logits", _vp), ("target_stride", _ll),
                ("ids", _vp), ("lp", _vp), ("lse", _vp),
                ("node_token", _vp), ("parent", _vp), ("depth", _vp), ("node_rank", _vp),
                ("score", _vp), ("anc", _vp), ("n_nodes", _vp),
                ("attn_out", _vp), ("attn_lse", _vp),
                ("target_argmax", _vp), ("path", _vp), ("accept_len", _vp),
                ("next_bonus", _vp), ("src_slot", _vp), ("dst_slot", _vp),
                ("new_prefix_len", _vp),
                ("ws", _vp), ("ws_bytes", _sz),
                ("gain_floor", _vp), ("sampling", ctypes.POINTER(Sampling)),
                ("tree_q_in", _vp), ("tree_k_in", _vp), ("tree_v_in", _vp), ("rope_theta", ctypes.c_double),
                ("target_hidden", _vp), ("lm_head", _vp), ("d_model", _i),
                ("stage_events", ctypes.POINTER(_vp))]


_SIGS = {
    "ddtree_topk_workspace_bytes": (_sz, [_i, _i, _i]),
    "ddtree_topk": (_i, [_vp, _i, _i, _i, _ll, _i, _vp, _vp, _vp, _vp, _sz, _vp]),
    "ddtree_build": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "ddtree_build_ex": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i,
                             _vp, _vp]),
    "ddtree_tree_kv_write": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, ctypes.POINTER(KVDesc), _vp, _i,
                                  ctypes.c_double, _vp, _vp, _vp]),
    "ddtree_lmhead_workspace_bytes": (_sz, [_i]),
    "ddtree_lmhead_argmax": (_i, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "ddtree_walk": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, ctypes.POINTER(KVDesc), _vp, _i,
                         _vp, _vp, _vp, _vp, _vp, _vp]),
    "ddtree_attn_workspace_bytes": (_sz, [ctypes.POINTER(KVDesc), _i]),
    "ddtree_tree_attn": (_i, [_vp, _vp, _vp, _i, ctypes.POINTER(KVDesc), _vp, _vp, _vp, _vp, _i,
                              _vp, _vp, _vp, _sz, _vp]),
    "ddtree_accept_workspace_bytes": (_sz, [_i, _i, _i]),
    "ddtree_accept": (_i, [_vp, _i, _i, _ll, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp,
                           ctypes.POINTER(KVDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "ddtree_accept_ex": (_i, [_vp, _i, _i, _ll, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp,
                              ctypes.POINTER(KVDesc), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                              ctypes.POINTER(Sampling), _vp, _sz, _vp]),
    "ddtree_round_workspace_bytes": (_sz, [ctypes.POINTER(RoundArgs)]),
    "ddtree_round": (_i, [ctypes.POINTER(RoundArgs), _vp]),
    "ddtree_round_launch_count": (_i, [ctypes.POINTER(RoundArgs)]),
    "ddtree_status_string": (ctypes.c_char_p, [_i]),
    "ddtree_device_status": (_i, [_vp, ctypes.POINTER(ctypes.c_uint)]),
    "ddtree_version": (_i, []),
    "ddtree_last_error": (ctypes.c_char_p, []),
    "ddtree_topk_static_ws": (_i, [_vp, _i, _i, _i, _ll, _i, _vp, _vp, _vp, _vp]),
    "ddtree_debug_attn_timeout": (_i, [ctypes.c_ulonglong, _i]),
    "ddtree_attn_plan": (_i, [ctypes.POINTER(KVDesc), _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]),
    "ddtree_round_host": (_i, [ctypes.POINTER(RoundArgs), _vp, _vp]),
    "ddtree_round_host_bytes": (_i, [ctypes.POINTER(RoundArgs), _vp, ctypes.POINTER(ctypes.c_ulonglong),
                                     ctypes.POINTER(ctypes.c_ulonglong)]),
}


def lib() -> ctypes.CDLL:
    """Load libddtree.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise DDTreeError(f"{_LIB_PATH} is missing: build it with "
                              "`python -m draft_tree_build_ddtree_b200.build_lib`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def _check(status: int, what: str):
    if status != 0:
        msg = lib().ddtree_status_string(status).decode()
        if status == 3:
            msg += f" [{lib().ddtree_last_error().decode()}]"
        raise DDTreeError(f"{what}: {msg} ({status})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise DDTreeError(f"{name} must be a CUDA tensor (no CPU path exists)")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise DDTreeError(f"unsupported dtype {t.dtype}")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _contig(t: torch.Tensor, name: str):
    _dev(t, name)
    if not t.is_contiguous():
        raise DDTreeError(f"{name} must be contiguous")


class Workspace:
    """Zero-filled device scratch that grows on demand (one per call site)."""

    def __init__(self):
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int, device) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != torch.device(device):
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        return self.buf


_ws = {"topk": Workspace(), "attn": Workspace(), "accept": Workspace(), "round": Workspace()}


def device_status() -> int:
    """Synchronise the current stream; return and clear the device status bits."""
    bits = ctypes.c_uint(0)
    _check(lib().ddtree_device_status(_stream(), ctypes.byref(bits)), "ddtree_device_status")
    return int(bits.value)


# ------------------------------------------------------------------ stage 1

def ddtree_topk(logits: torch.Tensor, K: int, ids=None, lp=None, lse=None, ws=None):
    """Top-K and log-softmax of every row of ``logits`` ([rows, V], last dim contiguous)."""
    _dev(logits, "logits")
    if logits.dim() != 2 or logits.stride(1) != 1:
        raise DDTreeError("logits must be [rows, V] with a contiguous last dim")
    rows, V = logits.shape
    dev = logits.device
    ids = torch.empty((rows, K), dtype=torch.int32, device=dev) if ids is None else ids
    lp = torch.empty((rows, K), dtype=torch.float32, device=dev) if lp is None else lp
    lse = torch.empty((rows,), dtype=torch.float32, device=dev) if lse is None else lse
    need = lib().ddtree_topk_workspace_bytes(rows, V, K)
    w = _ws["topk"].get(need, dev) if ws is None else ws
    _check(lib().ddtree_topk(_ptr(logits), _dtype_code(logits), rows, V, logits.stride(0), K,
                             _ptr(ids), _ptr(lp), _ptr(lse), _ptr(w), w.numel(), _stream()),
           "ddtree_topk")
    return ids, lp, lse


# ------------------------------------------------------------------ stage 2

@dataclasses.dataclass
class Tree:
    node_token: torch.Tensor
    parent: torch.Tensor
    depth: torch.Tensor
    node_rank: torch.Tensor
    score: torch.Tensor
    anc: torch.Tensor
    n_nodes: torch.Tensor


def alloc_tree(n_req: int, B: int, device) -> Tree:
    n = B + 1
    W = (n + 31) // 32
    i32 = dict(dtype=torch.int32, device=device)
    return Tree(torch.empty((n_req, n), **i32), torch.empty((n_req, n), **i32),
                torch.empty((n_req, n), **i32), torch.empty((n_req, n), **i32),
                torch.empty((n_req, n), dtype=torch.float32, device=device),
                torch.empty((n_req, n, W), **i32), torch.empty((n_req,), **i32))


BUILD_FORCE_HEAP = 0x1
BUILD_PATH_NAMES = {0: "enumeration", 1: "heap_registers_3", 2: "heap_registers_9", 3: "heap_tournament"}


def ddtree_build(ids: torch.Tensor, lp: torch.Tensor, root_token: torch.Tensor, B: int,
                 out: Optional[Tree] = None, gain_floor: Optional[torch.Tensor] = None,
                 flags: int = 0, build_path: Optional[torch.Tensor] = None) -> Tree:
    """Best-first tree of ``B`` nodes per request from [n_req, L, K] top-K tables.

    ``gain_floor`` (float32 [n_req], optional): adaptive budget, keep only the
    pops whose score exceeds it.  ``flags`` / ``build_path``: see
    ddtree_build_ex in include/ddtree.h.
    """
    for t, nm in ((ids, "ids"), (lp, "lp"), (root_token, "root_token")):
        _contig(t, nm)
    n_req, L, K = ids.shape
    t = alloc_tree(n_req, B, ids.device) if out is None else out
    if gain_floor is None and flags == 0 and build_path is None:
        _check(lib().ddtree_build(_ptr(ids), _ptr(lp), _ptr(root_token), n_req, L, K, B,
                                  _ptr(t.node_token), _ptr(t.parent), _ptr(t.depth), _ptr(t.node_rank),
                                  _ptr(t.score), _ptr(t.anc), _ptr(t.n_nodes), _stream()),
               "ddtree_build")
        return t
    if gain_floor is not None:
        _contig(gain_floor, "gain_floor")
        if gain_floor.dtype != torch.float32 or gain_floor.numel() != n_req:
            raise DDTreeError("gain_floor must be float32 [n_req]")
    if build_path is not None:
        _contig(build_path, "build_path")
    _check(lib().ddtree_build_ex(_ptr(ids), _ptr(lp), _ptr(root_token), n_req, L, K, B,
                                 _ptr(t.node_token), _ptr(t.parent), _ptr(t.depth), _ptr(t.node_rank),
                                 _ptr(t.score), _ptr(t.anc), _ptr(t.n_nodes), _ptr(gain_floor), int(flags),
                                 _ptr(build_path), _stream()),
           "ddtree_build_ex")
    return t


# ------------------------------------------------------------------ stage 3

def kv_desc(layers, n_req, Hq, Hkv, D, paged=False, s_max=0, num_blocks=0, max_blocks=0,
            scale=0.0) -> KVDesc:
    return KVDesc(layers, n_req, Hq, Hkv, D, float(scale), int(bool(paged)), int(s_max),
                  int(num_blocks), int(max_blocks))


def kv_desc_for(k_cache: torch.Tensor, n_req: int, Hq: int, block_table=None, scale=0.0) -> KVDesc:
    """Descriptor of a contiguous [layers, n_req, S, Hkv, D] cache or a paged
    [layers, blocks, 64, Hkv, D] pool with ``block_table`` [n_req, max_blocks]."""
    layers, a, b, Hkv, D = k_cache.shape
    if block_table is None:
        return kv_desc(layers, n_req, Hq, Hkv, D, False, s_max=b, scale=scale)
    return kv_desc(layers, n_req, Hq, Hkv, D, True, num_blocks=a,
                   max_blocks=block_table.shape[1], scale=scale)


def ddtree_tree_attn(q, k_cache, v_cache, kv: KVDesc, prefix_len, anc, n_nodes, B,
                     block_table=None, out=None, out_lse=None, ws=None):
    """Ancestor-only attention of the tree nodes; q is [layers, n_req, B+1, Hq, D]."""
    for t, nm in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache"), (prefix_len, "prefix_len"),
                  (anc, "anc"), (n_nodes, "n_nodes")):
        _contig(t, nm)
    out = torch.empty_like(q) if out is None else out
    need = lib().ddtree_attn_workspace_bytes(ctypes.byref(kv), B)
    w = _ws["attn"].get(need, q.device) if ws is None else ws
    _check(lib().ddtree_tree_attn(_ptr(q), _ptr(k_cache), _ptr(v_cache), _dtype_code(q),
                                  ctypes.byref(kv), _ptr(block_table), _ptr(prefix_len), _ptr(anc),
                                  _ptr(n_nodes), B, _ptr(out), _ptr(out_lse), _ptr(w), w.numel(),
                                  _stream()),
           "ddtree_tree_attn")
    return out, out_lse


ATTN_KERNELS = {0: "cuda_core", 1: "one_mtile", 2: "two_mtile"}


def attn_plan(kv: KVDesc, B: int, dtype: int = BF16, num_sms: int = 0):
    """(kernel name, key-range splits) that ddtree_tree_attn launches for this
    geometry; host-only.  num_sms = 0 plans for the current device."""
    k, sp = ctypes.c_int(-1), ctypes.c_int(-1)
    _check(lib().ddtree_attn_plan(ctypes.byref(kv), B, dtype, num_sms, ctypes.byref(k), ctypes.byref(sp)),
           "ddtree_attn_plan")
    return ATTN_KERNELS[k.value], sp.value


def ddtree_tree_kv_write(k_in, v_in, depth, n_nodes, prefix_len, kv: KVDesc, k_cache, v_cache, B,
                         rope_theta: float = 1e6, q_in=None, q_out=None, block_table=None):
    """Rotate the tree nodes' Q/K to position P + depth and write K/V into the
    cache tail (ddtree_tree_kv_write); q_out defaults to q_in (in place)."""
    for t, nm in ((k_in, "k_in"), (v_in, "v_in"), (depth, "depth"), (n_nodes, "n_nodes"),
                  (prefix_len, "prefix_len"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _contig(t, nm)
    if q_in is not None and q_out is None:
        q_out = q_in
    _check(lib().ddtree_tree_kv_write(_ptr(q_in), _ptr(q_out), _ptr(k_in), _ptr(v_in), _dtype_code(k_in),
                                      _ptr(depth), _ptr(n_nodes), _ptr(prefix_len), ctypes.byref(kv),
                                      _ptr(block_table), B, float(rope_theta), _ptr(k_cache), _ptr(v_cache),
                                      _stream()),
           "ddtree_tree_kv_write")
    return q_out


_ws["lmhead"] = Workspace()


def ddtree_lmhead_argmax(hidden: torch.Tensor, weight: torch.Tensor, out=None, out_max=None, ws=None):
    """Per-row argmax of hidden [rows, d] @ weight[V, d]^T without writing the logits."""
    _contig(hidden, "hidden")
    _contig(weight, "weight")
    if hidden.dtype != torch.bfloat16 or weight.dtype != torch.bfloat16:
        raise DDTreeError("hidden and weight must be bf16")
    rows, d = hidden.shape
    V = weight.shape[0]
    out = torch.empty((rows,), dtype=torch.int32, device=hidden.device) if out is None else out
    w = _ws["lmhead"].get(lib().ddtree_lmhead_workspace_bytes(rows), hidden.device) if ws is None else ws
    _check(lib().ddtree_lmhead_argmax(_ptr(hidden), _ptr(weight), rows, V, d, _ptr(out), _ptr(out_max), _ptr(w),
                                      w.numel(), _stream()), "ddtree_lmhead_argmax")
    return out


def ddtree_walk(target_token, node_token, parent, n_nodes, L, prefix_len, k_cache=None, v_cache=None,
                kv: Optional[KVDesc] = None, block_table=None, out: Optional["Accept"] = None, dtype=BF16):
    """The verifier walk + compaction from per-node target tokens [n_req, B+1]."""
    _contig(target_token, "target_token")
    n_req, n = target_token.shape
    a = alloc_accept(n_req, L, n - 1, target_token.device) if out is None else out
    _check(lib().ddtree_walk(_ptr(target_token), _ptr(node_token), _ptr(parent), _ptr(n_nodes), n_req, L, n - 1,
                             _ptr(prefix_len), _ptr(a.new_prefix_len), _ptr(k_cache), _ptr(v_cache),
                             ctypes.byref(kv) if kv is not None else None, _ptr(block_table), int(dtype),
                             _ptr(a.path), _ptr(a.accept_len), _ptr(a.next_bonus), _ptr(a.src_slot),
                             _ptr(a.dst_slot), _stream()), "ddtree_walk")
    return a


# ------------------------------------------------------------------ stage 4

@dataclasses.dataclass
class Accept:
    target_argmax: torch.Tensor
    path: torch.Tensor
    accept_len: torch.Tensor
    next_bonus: torch.Tensor
    src_slot: torch.Tensor
    dst_slot: torch.Tensor
    new_prefix_len: torch.Tensor


def alloc_accept(n_req: int, L: int, B: int, device) -> Accept:
    i32 = dict(dtype=torch.int32, device=device)
    return Accept(torch.empty((n_req, B + 1), **i32), torch.empty((n_req, L + 1), **i32),
                  torch.empty((n_req,), **i32), torch.empty((n_req,), **i32),
                  torch.empty((n_req, L + 1), **i32), torch.empty((n_req, L + 1), **i32),
                  torch.empty((n_req,), **i32))


def ddtree_accept(target_logits, node_token, parent, n_nodes, L, prefix_len,
                  k_cache=None, v_cache=None, kv: Optional[KVDesc] = None, block_table=None,
                  out: Optional[Accept] = None, ws=None, temperature: float = 0.0, seed: int = 0,
                  offset: int = 0) -> Accept:
    """Verifier walk over [n_req, B+1, V] target logits; compacts the KV in place.

    temperature <= 0: greedy (argmax); > 0: one draw per node from
    softmax(z / temperature), keyed by (seed, offset) (ddtree_accept_ex).
    """
    _dev(target_logits, "target_logits")
    if target_logits.dim() != 3 or target_logits.stride(2) != 1:
        raise DDTreeError("target_logits must be [n_req, B+1, V] with a contiguous last dim")
    n_req, n, V = target_logits.shape
    if target_logits.stride(0) != n * target_logits.stride(1):
        raise DDTreeError("target_logits rows must be evenly strided")
    B = n - 1
    a = alloc_accept(n_req, L, B, target_logits.device) if out is None else out
    need = lib().ddtree_accept_workspace_bytes(n_req, B, V)
    w = _ws["accept"].get(need, target_logits.device) if ws is None else ws
    samp = Sampling(float(temperature), int(seed) & (2 ** 64 - 1), int(offset) & (2 ** 64 - 1))
    _check(lib().ddtree_accept_ex(_ptr(target_logits), _dtype_code(target_logits), V,
                                  target_logits.stride(1), _ptr(node_token), _ptr(parent), _ptr(n_nodes),
                                  n_req, L, B, _ptr(prefix_len), _ptr(a.new_prefix_len),
                                  _ptr(k_cache), _ptr(v_cache),
                                  ctypes.byref(kv) if kv is not None else None, _ptr(block_table),
                                  _ptr(a.target_argmax), _ptr(a.path), _ptr(a.accept_len),
                                  _ptr(a.next_bonus), _ptr(a.src_slot), _ptr(a.dst_slot),
                                  ctypes.byref(samp), _ptr(w), w.numel(), _stream()),
           "ddtree_accept_ex")
    return a


# ------------------------------------------------------------------ the round

@dataclasses.dataclass
class RoundBuffers:
    """Device inputs and outputs of one round (all CUDA tensors)."""
    n_req: int
    L: int
    V: int
    K: int
    B: int
    kv: KVDesc
    drafter_logits: torch.Tensor      # [n_req, L, V]
    root_token: torch.Tensor          # [n_req]
    q: torch.Tensor                   # [layers, n_req, B+1, Hq, D]
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    block_table: Optional[torch.Tensor]
    prefix_len: torch.Tensor          # [n_req]
    target_logits: torch.Tensor       # [n_req, B+1, V]
    ids: torch.Tensor = None
    lp: torch.Tensor = None
    lse: torch.Tensor = None
    tree: Tree = None
    attn_out: torch.Tensor = None
    attn_lse: torch.Tensor = None
    acc: Accept = None
    ws: torch.Tensor = None
    gain_floor: Optional[torch.Tensor] = None   # float32 [n_req]: adaptive-budget floor of the build
    sampling: Optional[Sampling] = None         # temperature > 0 verification (None: greedy)
    tree_q_in: Optional[torch.Tensor] = None    # un-rotated tree Q/K/V: the round rotates and writes them
    tree_k_in: Optional[torch.Tensor] = None
    tree_v_in: Optional[torch.Tensor] = None
    rope_theta: float = 1e6
    target_hidden: Optional[torch.Tensor] = None   # [n_req*(B+1), d] bf16: argmax from the LM head instead
    lm_head: Optional[torch.Tensor] = None         # [V, d] bf16
    _args: RoundArgs = None

    def allocate_outputs(self):
        dev = self.drafter_logits.device
        rows = self.n_req * self.L
        self.ids = torch.empty((self.n_req, self.L, self.K), dtype=torch.int32, device=dev)
        self.lp = torch.empty((self.n_req, self.L, self.K), dtype=torch.float32, device=dev)
        self.lse = torch.empty((rows,), dtype=torch.float32, device=dev)
        self.tree = alloc_tree(self.n_req, self.B, dev)
        self.attn_out = torch.empty_like(self.q)
        self.attn_lse = torch.empty(self.q.shape[:-1], dtype=torch.float32, device=dev)
        self.acc = alloc_accept(self.n_req, self.L, self.B, dev)
        return self

    def args(self) -> RoundArgs:
        """The packed C argument struct (rebuilt when a buffer is swapped)."""
        a = RoundArgs()
        a.n_req, a.L, a.V, a.K, a.B = self.n_req, self.L, self.V, self.K, self.B
        a.dtype = _dtype_code(self.drafter_logits)
        a.kv = self.kv
        a.drafter_logits = _ptr(self.drafter_logits)
        a.drafter_stride = self.drafter_logits.stride(1)
        a.root_token = _ptr(self.root_token)
        a.q, a.k_cache, a.v_cache = _ptr(self.q), _ptr(self.k_cache), _ptr(self.v_cache)
        a.block_table = _ptr(self.block_table)
        a.prefix_len = _ptr(self.prefix_len)
        a.target_logits = _ptr(self.target_logits)
        a.target_stride = self.target_logits.stride(1)
        a.ids, a.lp, a.lse = _ptr(self.ids), _ptr(self.lp), _ptr(self.lse)
        t = self.tree
        a.node_token, a.parent, a.depth = _ptr(t.node_token), _ptr(t.parent), _ptr(t.depth)
        a.node_rank, a.score, a.anc, a.n_nodes = _ptr(t.node_rank), _ptr(t.score), _ptr(t.anc), _ptr(t.n_nodes)
        a.attn_out, a.attn_lse = _ptr(self.attn_out), _ptr(self.attn_lse)
        c = self.acc
        a.target_argmax, a.path, a.accept_len = _ptr(c.target_argmax), _ptr(c.path), _ptr(c.accept_len)
        a.next_bonus, a.src_slot, a.dst_slot = _ptr(c.next_bonus), _ptr(c.src_slot), _ptr(c.dst_slot)
        a.new_prefix_len = _ptr(c.new_prefix_len)
        a.gain_floor = _ptr(self.gain_floor)
        if self.sampling is not None:
            a.sampling = ctypes.pointer(self.sampling)
        a.tree_q_in, a.tree_k_in, a.tree_v_in = _ptr(self.tree_q_in), _ptr(self.tree_k_in), _ptr(self.tree_v_in)
        a.rope_theta = float(self.rope_theta)
        a.target_hidden, a.lm_head = _ptr(self.target_hidden), _ptr(self.lm_head)
        a.d_model = 0 if self.target_hidden is None else int(self.target_hidden.shape[-1])
        need = lib().ddtree_round_workspace_bytes(ctypes.byref(a))
        if need == 0:
            raise DDTreeError("invalid round geometry")
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.zeros(need, dtype=torch.uint8, device=self.drafter_logits.device)
        a.ws, a.ws_bytes = _ptr(self.ws), self.ws.numel()
        self._args = a
        return a


def ddtree_round(rb: RoundBuffers, args: Optional[RoundArgs] = None):
    """topk -> build -> tree attention -> accept on the current stream."""
    a = rb.args() if args is None else args
    _check(lib().ddtree_round(ctypes.byref(a), _stream()), "ddtree_round")
    return rb


STAGES = ("topk", "build", "tree_kv_write", "attn", "accept")


def ddtree_round_timed(rb: RoundBuffers) -> dict:
    """One round with stage events: {stage: ms} from the events the round
    records at its stage boundaries (synchronises the current stream)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(STAGES) + 1)]
    for e in evs:
        e.record()                          # creates the event
    arr = (ctypes.c_void_p * len(evs))(*[e.cuda_event for e in evs])
    a = rb.args()
    a.stage_events = ctypes.cast(arr, ctypes.POINTER(ctypes.c_void_p))
    _check(lib().ddtree_round(ctypes.byref(a), _stream()), "ddtree_round")
    evs[-1].synchronize()
    a.stage_events = None
    return {name: evs[i].elapsed_time(evs[i + 1]) for i, name in enumerate(STAGES)}


def ddtree_round_launch_count(rb: RoundBuffers, args: Optional[RoundArgs] = None) -> int:
    """Kernel launches one ddtree_round call makes with these buffers."""
    a = rb.args() if args is None else args
    n = lib().ddtree_round_launch_count(ctypes.byref(a))
    if n < 0:
        raise DDTreeError("invalid round geometry")
    return n


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
