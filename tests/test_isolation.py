"""The oracle and the CUDA path stay apart, and the product path has no fallback.

Static checks over the sources: the product package (the C-ABI library's
sources and its Python binding) and the shared input generators import nothing
from ``oracle/``; ``oracle/`` imports nothing from the product package; and
``bench.py`` reaches the oracle only inside its CPU-baseline / reference-arm
functions. A child process checks that the binding raises when the compiled
library is missing instead of falling back to anything else.
"""
import ast
import glob
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "sink_aware_sliding_head_b200")
ORACLE_FUNCS = {"oracle_sample", "oracle_decode_sample"}


def _imports(path):
    """(module, enclosing function or None) for every import in a Python file."""
    tree = ast.parse(open(path).read(), filename=path)
    out = []

    def visit(node, func):
        for child in ast.iter_child_nodes(node):
            f = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else func
            if isinstance(child, ast.Import):
                out.extend((a.name, func) for a in child.names)
            elif isinstance(child, ast.ImportFrom):
                out.append((child.module or "", func))
            visit(child, f)

    visit(tree, None)
    return out


def test_product_package_and_inputs_do_not_import_the_oracle():
    files = glob.glob(os.path.join(PKG, "**", "*.py"), recursive=True)
    files += glob.glob(os.path.join(ROOT, "flint_inputs", "*.py"))
    for f in files:
        for mod, _ in _imports(f):
            assert mod.split(".")[0] != "oracle", (f, mod)
    for f in glob.glob(os.path.join(PKG, "csrc", "*.cu*")):
        for line in open(f):
            if line.lstrip().startswith("#include"):
                assert "oracle" not in line, (f, line)


def test_oracle_does_not_import_the_product_package():
    for f in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        for mod, _ in _imports(f):
            assert not mod.startswith("sink_aware_sliding_head_b200"), (f, mod)
        assert "libflint_attn" not in open(f).read(), f


def test_bench_reaches_the_oracle_only_in_its_cpu_baseline_functions():
    uses = [(mod, func) for mod, func in _imports(os.path.join(ROOT, "bench.py"))
            if mod.split(".")[0] == "oracle"]
    assert uses, "bench.py has a CPU-baseline leg"
    for mod, func in uses:
        assert func in ORACLE_FUNCS, (mod, func)


def test_binding_raises_without_the_library():
    code = ("import sink_aware_sliding_head_b200.flint_attn as fa\n"
            "try:\n"
            "    fa.load_library('/nonexistent/libflint_attn.so')\n"
            "except ImportError:\n"
            "    print('raised')\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.stdout.strip() == "raised", r.stdout + r.stderr
