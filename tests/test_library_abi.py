"""The C-ABI library builds, loads and exports what include/ddtree.h declares.

CPU only: no call here launches a kernel.  Argument checks run on the host
before any CUDA call, so invalid arguments are rejected without a device.
"""
import ctypes
import os
import re

import pytest

import draft_tree_build_ddtree_b200 as dd
from draft_tree_build_ddtree_b200 import build_lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


def declared_functions():
    names = []
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w \*]*?\b(ddtree_\w+)\s*\(", src, flags=re.M):
            names.append(m.group(1))
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return dd.lib()


def test_header_declares_the_round_entry_points():
    names = declared_functions()
    for n in ("ddtree_topk", "ddtree_build", "ddtree_tree_attn", "ddtree_accept", "ddtree_round"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_covers_every_declared_symbol():
    assert set(declared_functions()) <= set(dd.exported_symbols())


def test_status_strings(lib):
    assert lib.ddtree_status_string(0) == b"ok"
    assert lib.ddtree_status_string(1) == b"invalid argument"
    assert lib.ddtree_version() >= 100


def test_host_validation_rejects_bad_arguments(lib):
    INVALID = 1
    # null logits
    assert lib.ddtree_topk(None, 0, 16, 1000, 1000, 8, None, None, None, None, 0, None) == INVALID
    # K > V
    p = ctypes.c_void_p(16)
    assert lib.ddtree_topk(p, 0, 1, 8, 8, 9, p, p, None, p, 1 << 20, None) == INVALID
    # row stride not a multiple of 16 bytes
    assert lib.ddtree_topk(p, 0, 1, 1001, 1001, 8, p, p, None, p, 1 << 20, None) == INVALID
    # misaligned logits pointer
    assert lib.ddtree_topk(ctypes.c_void_p(18), 0, 1, 1000, 1000, 8, p, p, None, p, 1 << 20,
                           None) == INVALID
    # budget above the limit; L above the limit
    assert lib.ddtree_build(p, p, p, 1, 16, 64, 1025, p, p, p, p, p, p, p, None) == INVALID
    assert lib.ddtree_build(p, p, p, 1, 33, 64, 64, p, p, p, p, p, p, p, None) == INVALID
    # accept: output aliasing its input
    kv = dd.kv_desc(1, 1, 32, 4, 128, s_max=4096)
    assert lib.ddtree_accept(p, 0, 1000, 1000, p, p, p, 1, 16, 64, p, p, None, None,
                             ctypes.byref(kv), None, None, None, None, None, None, None, p,
                             1 << 20, None) == INVALID
    # attention: Hq not a multiple of Hkv; unsupported head dim
    bad = dd.kv_desc(1, 1, 30, 4, 128, s_max=4096)
    assert lib.ddtree_tree_attn(p, p, p, 0, ctypes.byref(bad), None, p, p, p, 64, p, None, p,
                                1 << 20, None) == INVALID
    odd = dd.kv_desc(1, 1, 32, 4, 96, s_max=4096)
    assert lib.ddtree_tree_attn(p, p, p, 0, ctypes.byref(odd), None, p, p, p, 64, p, None, p,
                                1 << 20, None) == 2


def test_cpu_tensors_are_refused():
    import torch
    with pytest.raises(dd.DDTreeError):
        dd.ddtree_topk(torch.zeros(2, 64), 4)


def test_round_launch_count_is_host_only(lib):
    """The round's launch plan is computed on the host from sizes alone (no
    pointer is read): top-K, build, attention (+ combine when the key range
    is split), argmax (+ walk launch above two cache layers)."""
    def args(layers, P, dtype=0, n_req=1, B=64, D=128):
        a = dd.RoundArgs()
        a.n_req, a.L, a.V, a.K, a.B = n_req, 16, 151936, 64, B
        a.dtype = dtype
        a.kv = dd.kv_desc(layers, n_req, 32, 4, D, s_max=(P + B + 1 + 63) // 64 * 64)
        return a

    def count(a):
        return lib.ddtree_round_launch_count(ctypes.byref(a))

    # without a device the library plans for 148 SMs; these plans hold for any B200
    assert count(args(1, 2048)) == 5            # b64_p2k: 20 units split over the SMs -> combine
    assert count(args(48, 8192, B=256)) == 5    # 3264 units fill the GPU (no combine); 48 layers -> walk launch
    assert count(args(1, 2048, dtype=1)) == 4   # fp32: SIMT attention, no split
    bad = args(1, 2048)
    bad.n_req = 0
    assert count(bad) == -1


def _align256(x):
    return (x + 255) // 256 * 256


def test_launch_plans_from_sizes(lib):
    """The host-side plans (148 SMs without a device) behind the workspace
    sizes: b64_p2k top-K cuts each of its 16 bf16 rows into 9 chunks (one
    wave of 144 CTAs) with K + K candidate slots each; the b64_p2k attention splits
    its 20 units (4 KV heads x 5 M-tiles) 7 ways over 128-key tiles; the
    32k-prefix sweep splits its M-tile pairs; the 48-layer and 32-request
    workloads fill the GPU unsplit."""
    rows, V, K = 16, 151936, 64
    cap = 2 * K

    def topk_ws(cpr):
        return (_align256(rows * 4) + _align256(rows * cpr * 16) + 2 * _align256(rows * cpr * 4)
                + _align256(rows * cpr * cap * 8))
    # the query covers either dtype: bf16 rows take 9 chunks (one wave of
    # 144 CTAs); fp32 rows need 13 (at most 6 x 512 x 16 bytes staged per CTA)
    assert lib.ddtree_topk_workspace_bytes(rows, V, K) == max(topk_ws(9), topk_ws(13)) == topk_ws(13)

    kv2 = dd.kv_desc(1, 1, 32, 4, 128, s_max=2176)
    slots = 20 * 7
    assert lib.ddtree_attn_workspace_bytes(ctypes.byref(kv2), 64) == \
        _align256(slots * 128 * 128 * 4) + _align256(slots * 128 * 8)
    assert dd.attn_plan(kv2, 64, num_sms=148) == ("one_mtile", 7)
    # sweep_p32k at B = 64: the two-M-tile kernel, 4 KV heads x 3 M-tile pairs
    # split 12 ways; partials per (M-tile, split): 4 x 5 x 12
    kv5 = dd.kv_desc(1, 1, 32, 4, 128, s_max=32896)
    assert dd.attn_plan(kv5, 64, num_sms=148) == ("two_mtile", 12)
    slots = 4 * 5 * 12
    assert lib.ddtree_attn_workspace_bytes(ctypes.byref(kv5), 64) == \
        _align256(slots * 128 * 128 * 4) + _align256(slots * 128 * 8)
    # bf16 with D = 64 always takes the two-M-tile kernel: b64_p2k's shape
    # with D = 64 splits its 12 M-tile pairs twice (8 key tiles each at least)
    kv64 = dd.kv_desc(1, 1, 32, 4, 64, s_max=2176)
    assert dd.attn_plan(kv64, 64, num_sms=148) == ("two_mtile", 2)
    slots = 4 * 5 * 2
    assert lib.ddtree_attn_workspace_bytes(ctypes.byref(kv64), 64) == \
        _align256(slots * 128 * 64 * 4) + _align256(slots * 128 * 8)
    kv3 = dd.kv_desc(48, 1, 32, 4, 128, s_max=8512)
    assert lib.ddtree_attn_workspace_bytes(ctypes.byref(kv3), 256) == 0
    assert dd.attn_plan(kv3, 256, num_sms=148) == ("two_mtile", 1)
    assert dd.attn_plan(kv3, 256, dd.F32, num_sms=148) == ("cuda_core", 1)
    kv4 = dd.kv_desc(1, 32, 32, 4, 128, paged=True, num_blocks=4096, max_blocks=258)
    assert lib.ddtree_attn_workspace_bytes(ctypes.byref(kv4), 64) == 0
    assert dd.attn_plan(kv4, 64, num_sms=148) == ("two_mtile", 1)
    # accept: composite slots, argmax, one ticket per request
    n = 65
    assert lib.ddtree_accept_workspace_bytes(32, 64, V) == \
        _align256(32 * n * 8) + _align256(32 * n * 4) + _align256(32 * 4)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No CPU fallback: without libddtree.so every call raises."""
    monkeypatch.setattr(dd, "_LIB_PATH", str(tmp_path / "libddtree.so"))
    monkeypatch.setattr(dd, "_lib", None)
    with pytest.raises(dd.DDTreeError):
        dd.lib()
