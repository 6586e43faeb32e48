"""The product path never reaches the oracle and has no CPU fallback (CPU only).

The oracle is test infrastructure: the package's Python modules, the CUDA
sources and the public header must not import, include, load or name it, and
the binding must fail loudly when the CUDA library is missing instead of
computing anything itself.
"""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "combine_top_route_counting_b200")


def _py_files():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_package_python_never_imports_the_oracle():
    for path in _py_files():
        tree = ast.parse(open(path).read(), filename=path)
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            else:
                continue
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names), path


def test_cuda_sources_and_header_never_name_the_oracle():
    srcs = [os.path.join(ROOT, "include", "moe.h")]
    csrc = os.path.join(PKG, "csrc")
    srcs += [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh"))]
    for path in srcs:
        text = open(path).read()
        assert not re.search(r"#include\s+[<\"][^>\"]*oracle", text), path
        assert "moe_oracle" not in text and "libmoe_oracle" not in text, path


def test_binding_exports_only_library_entry_points():
    """Every public moe_* function of the binding forwards to the C entry of the
    same name (argument marshalling only): its body calls load().<same name>."""
    from combine_top_route_counting_b200 import moe
    src = open(os.path.join(PKG, "moe.py")).read()
    tree = ast.parse(src)
    funcs = [n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name.startswith("moe_")]
    assert funcs
    for fn in funcs:
        body = ast.get_source_segment(src, fn)
        assert f"load().{fn.name}(" in body, fn.name
        assert fn.name in moe.exported_symbols(), fn.name


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    from combine_top_route_counting_b200 import moe
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError):
        moe.load()


def test_bench_and_entry_touch_the_oracle_only_in_their_baseline_legs():
    """bench.py imports the oracle only inside its CPU-baseline / reference
    functions; __graft_entry__ only inside smoke() and build()'s checker build."""
    src = open(os.path.join(ROOT, "bench.py")).read()
    tree = ast.parse(src)
    allowed = {"oracle_sample", "run_reference"}
    for node in ast.walk(tree):
        if isinstance(node, (ast.FunctionDef,)):
            seg = ast.get_source_segment(src, node)
            if re.search(r"^\s*(import oracle|from oracle)", seg, re.M):
                assert node.name in allowed, node.name
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for n in top:
        names = [a.name for a in n.names] if isinstance(n, ast.Import) else [n.module or ""]
        assert not any(x.startswith("oracle") for x in names)
