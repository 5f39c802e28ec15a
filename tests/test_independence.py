"""The oracle and the CUDA path share no code.

Static checks on the sources (CPU only): the oracle imports only the
standard library and numpy; nothing in the package, its CUDA sources or its
C header refers to the oracle; the only module both sides' tests use,
datagen, imports neither.
"""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "draft_tree_build_ddtree_b200")


def imported_modules(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level:
                mods.add("." + (node.module or ""))
            elif node.module:
                mods.add(node.module.split(".")[0])
    return mods


def test_oracle_imports_only_stdlib_and_numpy():
    allowed = {"__future__", "dataclasses", "heapq", "itertools", "typing", "numpy", "math", "functools",
               "collections", "."}
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        mods = imported_modules(path)
        assert mods <= allowed | {".ddtree_oracle"}, (path, mods - allowed)


def test_package_never_refers_to_the_oracle():
    for path in glob.glob(os.path.join(PKG, "*.py")):
        assert "oracle" not in imported_modules(path), path
    for path in (glob.glob(os.path.join(PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*.h"))):
        src = open(path, errors="replace").read()
        assert not re.search(r"#\s*include\s*[<\"][^>\"]*oracle", src), path


def test_datagen_holds_no_method_code():
    mods = imported_modules(os.path.join(PKG, "datagen.py"))
    assert "oracle" not in mods
    assert not any(m.startswith(".") for m in mods), mods   # nothing from the package's compute path
