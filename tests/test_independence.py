"""The oracle and the CUDA path share no code, on CPU: no module of the
library package imports the oracle, no oracle module imports the library,
the CUDA sources include nothing from the oracle, and bench.py reaches the
oracle only inside its CPU-baseline / reference functions."""

import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _py_files(rel_dir):
    for dirpath, _, files in os.walk(os.path.join(ROOT, rel_dir)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read())
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name.split(".")[0], node
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            yield node.module.split(".")[0], node


def test_library_never_imports_the_oracle():
    for path in _py_files("few_step_dit_b200"):
        for mod, _ in _imports(path):
            assert mod != "oracle", path


def test_oracle_never_imports_the_library():
    for path in _py_files("oracle"):
        for mod, _ in _imports(path):
            assert mod not in ("few_step_dit_b200", "bench"), path


def test_cuda_sources_include_nothing_from_the_oracle():
    csrc = os.path.join(ROOT, "few_step_dit_b200", "csrc")
    for f in os.listdir(csrc):
        if f.endswith((".cu", ".cuh", ".h")):
            text = open(os.path.join(csrc, f), encoding="utf-8").read()
            for inc in re.findall(r'#include\s+"([^"]+)"', text):
                assert "oracle" not in inc, (f, inc)


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path, encoding="utf-8").read())
    # top-level imports: no oracle
    for node in tree.body:
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert not any(n.split(".")[0] == "oracle" for n in names)
    # every oracle import sits inside the CPU-baseline sample or the reference arm
    allowed = {"oracle_sample", "oracle_tiny", "run_reference"}
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            if isinstance(node, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in node.names):
                assert fn.name in allowed, fn.name
            if isinstance(node, ast.ImportFrom) and (node.module or "").split(".")[0] == "oracle":
                assert fn.name in allowed, fn.name
