"""The bounds-checked build (libddtree_debug.so, -DDDTREE_DEBUG): a full
round on the b64_p2k and paged batch workloads, in a child process that
loads it, flags nothing (no DDTREE_STATUS_BOUNDS) and matches the oracle
exactly like the release build."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))

CHILD = r"""
import sys
sys.path.insert(0, {tests!r})
import draft_tree_build_ddtree_b200 as dd
assert dd._LIB_PATH.endswith("libddtree_debug.so"), dd._LIB_PATH
import torch
from draft_tree_build_ddtree_b200 import datagen
from test_gpu_round import make_round, check_round
for cfg, over, sample in ((2, {{}}, {{}}), (4, dict(N=6), dict(nodes=[0, 3, 64], heads=[0, 31])),
                          (3, dict(layers=4), dict(layers=[0, 3], nodes=[0, 1, 256], heads=[0, 31]))):
    w = datagen.workload(cfg, **over)
    rb, h = make_round(w)
    dd.ddtree_round(rb)
    torch.cuda.synchronize()
    check_round(w, rb, h, **sample)        # includes: device status 0 (no bounds flag)
print("debug build ok")
"""


def test_debug_build_round_is_clean_and_exact():
    root = os.path.dirname(HERE)
    lib = os.path.join(root, "draft_tree_build_ddtree_b200", "libddtree_debug.so")
    assert os.path.exists(lib), "build it with build_lib.build(debug=True)"
    env = dict(os.environ, DDTREE_LIBRARY="debug", PYTHONPATH=root)
    r = subprocess.run([sys.executable, "-c", CHILD.format(tests=HERE)], env=env, capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert "debug build ok" in r.stdout
