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
