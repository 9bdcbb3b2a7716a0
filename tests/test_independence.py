"""The oracle and the CUDA path stay independent (static checks, no GPU).

The package never imports the oracle and the oracle never imports the package;
the C oracle includes only standard headers; the benchmark touches the oracle
only inside its CPU baseline leg; the seeded input generator holds no part of
the method's arithmetic beyond the e4m3 encoding of its inputs.
"""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    """Top-level module names imported anywhere in a Python file, with the
    enclosing function of each import (None at module level)."""
    tree = ast.parse(open(path).read(), filename=path)
    found = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import):
                found.extend((a.name.split(".")[0], func) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                if child.level == 0 and child.module:
                    found.append((child.module.split(".")[0], func))
            visit(child, f)

    visit(tree, None)
    return found


def test_package_never_imports_the_oracle():
    files = glob.glob(os.path.join(ROOT, "block_sparse_prefill_b200", "**", "*.py"), recursive=True)
    assert files
    for f in files:
        assert "oracle" not in {m for m, _ in _imports(f)}, f


def test_oracle_never_imports_the_package_or_the_generator():
    for f in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        mods = {m for m, _ in _imports(f)}
        assert "block_sparse_prefill_b200" not in mods and "workloads" not in mods, f


def test_c_oracle_includes_only_standard_headers():
    src = open(os.path.join(ROOT, "oracle", "fp2_oracle.c")).read()
    includes = re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', src)
    assert set(includes) <= {"math.h", "stdint.h", "stdlib.h", "string.h"}, includes


def test_cuda_sources_never_include_the_oracle():
    for f in glob.glob(os.path.join(ROOT, "block_sparse_prefill_b200", "csrc", "*")):
        assert "oracle" not in open(f).read().lower(), f


def test_bench_uses_the_oracle_only_in_its_cpu_baseline_leg():
    uses = [func for m, func in _imports(os.path.join(ROOT, "bench.py")) if m == "oracle"]
    assert uses and set(uses) == {"cpu_baseline"}, uses


def test_generator_holds_no_method_arithmetic():
    """The seeded generator shares no estimator, threshold or attention step with
    either side: no softmax, exponential threshold or block-score code."""
    src = "".join(open(f).read() for f in glob.glob(os.path.join(ROOT, "workloads", "*.py")))
    for pattern in (r"softmax\(", r"logsumexp\(", r"kept_idx", r"kept_cnt", r"log\(alpha", r"block_means\("):
        assert not re.search(pattern, src), pattern
