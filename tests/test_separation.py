"""The CUDA path and the oracle stay apart (no shared code, no fallback).

* Nothing in the product package (the binding, the build script, the CUDA
  sources) imports, includes or loads the oracle.
* The oracle and the input generator import neither the package nor the
  library, and load no native code.
* bench.py reaches the oracle only inside its CPU-baseline and reference
  functions, never at import time.
* The binding refuses to load without the in-tree library: there is no
  Python or CPU fallback to fall through to.
"""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sparse_linear_hybrid_top_b200")


def _files(folder, exts):
    for base, _, names in os.walk(folder):
        if "_build" in base or "__pycache__" in base:
            continue
        for n in names:
            if n.endswith(exts):
                yield os.path.join(base, n)


def test_package_never_touches_the_oracle():
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|#\s*include\s+[<\"].*oracle)", re.M)
    hits = [p for p in _files(PKG, (".py", ".cu", ".cuh", ".h", ".cpp"))
            if pat.search(open(p, encoding="utf-8").read())]
    assert hits == []


@pytest.mark.parametrize("folder", ["oracle", "synth"])
def test_oracle_and_generator_use_no_product_code(folder):
    pat = re.compile(r"sparse_linear_hybrid_top_b200|libsalad|\bctypes\b|\bcdll\b", re.I)
    hits = [p for p in _files(os.path.join(ROOT, folder), (".py",))
            if pat.search(open(p, encoding="utf-8").read())]
    assert hits == []


def test_bench_imports_the_oracle_only_inside_functions():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    for node in tree.body:   # module level only
        if isinstance(node, ast.Import):
            assert all(a.name.split(".")[0] != "oracle" for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            assert (node.module or "").split(".")[0] != "oracle"


def test_binding_refuses_to_load_without_the_library(monkeypatch):
    import sparse_linear_hybrid_top_b200 as salad
    monkeypatch.setattr(salad, "LIB_PATH", os.path.join(PKG, "does-not-exist", "libsalad.so"))
    with pytest.raises(ImportError):
        salad._load()
