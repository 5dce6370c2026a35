"""The oracle stays test infrastructure: no module of the package imports it, and bench.py
imports it only inside its CPU-baseline and reference legs (checked on the source, no GPU)."""
import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "rotated_bit_dit_b200")
BENCH_ORACLE_LEGS = {"oracle_sample", "cpu_baseline", "run_reference"}


def oracle_imports(tree: ast.AST):
    """(enclosing function or None, line) of every import of the oracle package."""
    found = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.append((func, child.lineno))
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.append((func, child.lineno))
            visit(child, f)

    visit(tree, None)
    return found


def test_package_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith(".py"):
                path = os.path.join(dirpath, f)
                tree = ast.parse(open(path).read(), path)
                assert not oracle_imports(tree), path


def test_bench_imports_the_oracle_only_in_its_baseline_legs():
    path = os.path.join(ROOT, "bench.py")
    found = oracle_imports(ast.parse(open(path).read(), path))
    assert found, "the CPU-baseline leg is expected to use the oracle"
    for func, line in found:
        assert func in BENCH_ORACLE_LEGS, f"bench.py:{line} imports the oracle in {func}"


def test_package_fails_loudly_without_the_library(tmp_path, monkeypatch):
    """With no built library and building disabled, loading raises, and an entry point whose
    library cannot be loaded raises too (no CPU fallback)."""
    from rotated_bit_dit_b200 import _binding as B

    monkeypatch.setattr(B, "_LIB", None)
    monkeypatch.setattr(B, "lib_path", lambda: str(tmp_path / "missing" / "librbd.so"))
    with pytest.raises(RuntimeError):
        B.load(build_if_missing=False)

    def missing(build_if_missing=True):
        raise RuntimeError("librbd.so not built")

    monkeypatch.setattr(B, "load", missing)
    with pytest.raises(RuntimeError):
        B.rbd_version()


def test_tensor_on_another_device_is_refused_before_any_launch(monkeypatch):
    """Every kernel runs on the current device, so a pointer to another GPU's memory must be
    refused on the host (it would otherwise be dereferenced by the wrong GPU).  Host-side
    only: a stand-in tensor and a stand-in current device, no launch."""
    import torch
    from rotated_bit_dit_b200 import _binding as B

    class FakeCudaTensor:
        is_cuda = True

        def __init__(self, index):
            self.device = torch.device("cuda", index)

        def data_ptr(self):
            return 0x1000

    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert B._ptr(FakeCudaTensor(0)).value == 0x1000
    with pytest.raises(ValueError, match="cuda:1"):
        B._ptr(FakeCudaTensor(1))
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    assert B._ptr(FakeCudaTensor(1)).value == 0x1000
    with pytest.raises(ValueError):
        B._ptr(FakeCudaTensor(0))
