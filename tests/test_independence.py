"""The oracle and the CUDA path stay apart, and the product path has no CPU
fallback: the package, its kernels and the shared workload module import or
include nothing of the oracle; the oracle imports nothing of the package;
bench.py reaches the oracle only from the host-core baseline; the binding
raises when the library is missing."""
import ast
import os
import re

import pytest

from tests.conftest import ROOT

PKG = os.path.join(ROOT, "sink_window_attention_b200")


def _py_files(d):
    for base, _, files in os.walk(d):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def _imported_modules(path):
    tree = ast.parse(open(path).read(), path)
    mods = []
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods += [a.name for a in node.names]
        elif isinstance(node, ast.ImportFrom) and node.module:
            mods.append(node.module)
    return mods


def test_package_and_workloads_never_import_the_oracle():
    files = list(_py_files(PKG)) + list(_py_files(os.path.join(ROOT, "swa_workloads")))
    assert files
    for f in files:
        for m in _imported_modules(f):
            assert not (m == "oracle" or m.startswith("oracle.")), (f, m)


def test_kernels_include_nothing_outside_the_package_and_the_header():
    csrc = os.path.join(PKG, "csrc")
    for f in os.listdir(csrc):
        if not f.endswith((".cu", ".cuh", ".h")):
            continue
        for inc in re.findall(r'#include\s+"([^"]+)"', open(os.path.join(csrc, f)).read()):
            target = os.path.normpath(os.path.join(csrc, inc))
            assert target.startswith(PKG + os.sep) or target == os.path.join(ROOT, "include", "ll_api.h"), (f, inc)


def test_oracle_never_imports_the_package():
    for f in _py_files(os.path.join(ROOT, "oracle")):
        for m in _imported_modules(f):
            assert not m.startswith("sink_window_attention_b200"), (f, m)
            assert m not in ("torch", "ctypes"), (f, m)


def test_bench_reaches_the_oracle_only_from_the_host_core_baseline():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    for node in tree.body:                   # no module-level import of the oracle
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert not any(n == "oracle" or n.startswith("oracle.") for n in names)
    users = set()

    class Scopes(ast.NodeVisitor):
        def __init__(self):
            self.stack = []

        def visit_scope(self, node):
            self.stack.append(node.name)
            self.generic_visit(node)
            self.stack.pop()

        visit_FunctionDef = visit_ClassDef = visit_scope

        def visit_Import(self, node):
            if any(a.name == "oracle" or a.name.startswith("oracle.") for a in node.names):
                users.add(".".join(self.stack))

        def visit_ImportFrom(self, node):
            if (node.module or "") == "oracle" or (node.module or "").startswith("oracle."):
                users.add(".".join(self.stack))

    Scopes().visit(tree)
    assert users == {"OracleStep.__init__"}, users


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    import sink_window_attention_b200 as swa
    monkeypatch.setattr(swa, "_lib", None)
    monkeypatch.setattr(swa, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        swa.lib()
