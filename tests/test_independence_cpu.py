"""The oracle and the product share no code: the package, its CUDA sources and the C
header never name the oracle; the oracle never imports the package or includes its
headers; only the seeded input generator (no arithmetic of the method) serves both."""
import os
import re

import pytest

pytestmark = pytest.mark.cpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "ternary_weight_bit_absmean_b200")


def _files(top, exts):
    for dirpath, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(dirpath, n)


def test_product_never_reaches_the_oracle():
    for path in list(_files(PKG, (".py", ".cu", ".cuh", ".h"))) + [os.path.join(ROOT, "include", "bitlinear.h")]:
        text = open(path).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), path
        assert "bitlinear_oracle" not in text and "oracle/" not in text, path


def test_oracle_never_reaches_the_product():
    for path in _files(os.path.join(ROOT, "oracle"), (".py", ".c", ".h")):
        text = open(path).read()
        assert "ternary_weight_bit_absmean_b200" not in text, path
        assert not re.search(r'#include\s+"(bl_|bitlinear)', text), path
        assert "libbitlinear" not in text, path


def test_input_generator_holds_no_method_arithmetic():
    """synth.py draws numbers and names shapes: none of the method's operations (the
    absmean scale, rounding or clipping to codes, the absmax scale, packing)."""
    import ast
    tree = ast.parse(open(os.path.join(PKG, "synth.py")).read())
    for node in ast.walk(tree):  # drop docstrings
        if isinstance(node, (ast.Module, ast.FunctionDef, ast.ClassDef)) and node.body and \
                isinstance(node.body[0], ast.Expr) and isinstance(getattr(node.body[0], "value", None), ast.Constant):
            node.body = node.body[1:] or [ast.Pass()]
    code = ast.unparse(tree)
    for pat in (r"torch\.round", r"\.round\(", r"\.clamp\(", r"\.clip\(", r"abs\(\)\.mean", r"\.amax\(",
                r"\b127\b", r"0x[0-9A-Fa-f]+"):
        assert not re.search(pat, code), pat


def test_benchmark_uses_the_oracle_only_in_its_cpu_legs():
    text = open(os.path.join(ROOT, "bench.py")).read()
    lines = [i for i, line in enumerate(text.splitlines()) if re.search(r"\boracle\b", line) and "import" in line]
    assert lines, "the CPU baseline leg imports the oracle"
    funcs = [m.start() for m in re.finditer(r"^def (\w+)", text, re.M)]
    names = re.findall(r"^def (\w+)", text, re.M)
    owners = set()
    for i in lines:
        pos = sum(len(x) + 1 for x in text.splitlines()[:i])
        owner = max((f, n) for f, n in zip(funcs, names) if f <= pos)[1]
        owners.add(owner)
    assert owners <= {"cpu_baseline", "run_reference", "oracle_sample", "_oracle_step"}, owners
