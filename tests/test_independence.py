"""The oracle and the CUDA path share no code, and the product never reaches
the oracle (no GPU)."""

import ast
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _imports(path):
    tree = ast.parse(open(path, encoding="utf-8").read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d):
    for base, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_oracle_imports_nothing_from_the_product():
    for f in _py_files("oracle"):
        assert "exact_attention_120_b200" not in _imports(f), f


def test_product_never_imports_the_oracle():
    for f in _py_files("exact_attention_120_b200"):
        assert "oracle" not in _imports(f), f
    for base, _, files in os.walk(os.path.join(ROOT, "exact_attention_120_b200")):
        for fn in files:
            if fn.endswith((".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(base, fn), encoding="utf-8").read()
                assert "oracle" not in text.lower(), fn


def test_bench_reaches_the_oracle_only_from_its_cpu_legs():
    """bench.py imports the oracle only inside the functions that time it on
    the host (the CPU baseline and the reference arm's oracle samples), never
    at module level or on the GPU path."""
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"oracle_sample", "bwd_oracle_sample", "cpu_baseline"}

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            name = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                assert name in allowed, f"bench.py imports the oracle in {name!r} (line {child.lineno})"
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                assert name in allowed, f"bench.py imports the oracle in {name!r} (line {child.lineno})"
            visit(child, name)

    visit(tree, None)
