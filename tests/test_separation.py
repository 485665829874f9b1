"""Static checks that the CUDA path and the oracle stay independent.

The product package (the C ABI, its kernels and the binding) never imports,
links or includes anything under oracle/; the oracle never imports the
package or includes its headers; the seeded input generators both sides use
hold none of the method's arithmetic (no transform, no convolution); and
bench.py reaches the oracle only from its CPU-baseline sampler and the
reference arm."""
import ast
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "fft_long_convolution_causal_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _files(top, exts):
    for d, _, names in os.walk(top):
        for n in names:
            if n.endswith(exts):
                yield os.path.join(d, n)


def test_product_never_touches_the_oracle():
    pat = re.compile(r"\boracle\b.*import|import\s+oracle|from\s+oracle|liboracle|oracle/|fftconv_oracle")
    for f in _files(PKG, (".py", ".cu", ".cuh", ".h", ".c")):
        for i, line in enumerate(open(f, encoding="utf-8"), 1):
            assert not pat.search(line), f"{os.path.relpath(f, ROOT)}:{i}: {line.strip()}"


def test_oracle_never_touches_the_product():
    """Imports of the Python side and includes / dynamic loads of the C side."""
    for f in _files(ORACLE, (".py",)):
        src = open(f, encoding="utf-8").read()
        for node in ast.walk(ast.parse(src)):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            for n in names:
                assert not n.startswith("fft_long_convolution_causal_b200"), f"{f}: imports {n}"
        assert "libfftconv" not in src, f
    for f in _files(ORACLE, (".c", ".h")):
        for i, line in enumerate(open(f, encoding="utf-8"), 1):
            code = line.strip()
            if code.startswith("#include") or "dlopen" in code:
                assert not re.search(r"fftconv\.h|csrc|plan\.h|tables\.h|\.cuh|libfftconv", code), \
                    f"{os.path.relpath(f, ROOT)}:{i}: {code}"


def test_input_generators_hold_no_method_arithmetic():
    src = open(os.path.join(PKG, "workloads.py"), encoding="utf-8").read()
    tree = ast.parse(src)
    for node in ast.walk(tree):
        if isinstance(node, ast.Attribute):
            assert node.attr not in ("fft", "rfft", "irfft", "ifft", "fft2", "rfft2", "convolve", "correlate",
                                     "fftconvolve"), f"workloads.py uses {node.attr}"
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] + ([node.module] if isinstance(node, ast.ImportFrom) else [])
            for n in names:
                assert n and not n.split(".")[0] in ("scipy", "oracle", "torch"), f"workloads.py imports {n}"


def test_bench_reaches_the_oracle_only_from_its_baselines():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    allowed = {"OracleSampler", "cpu_oracle_rate", "main_reference"}
    for top in tree.body:
        for node in ast.walk(top):
            imported = []
            if isinstance(node, ast.Import):
                imported = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                imported = [node.module or ""]
            if any(n.split(".")[0] == "oracle" for n in imported):
                name = getattr(top, "name", None)
                assert name in allowed, f"bench.py imports the oracle in {name or 'module scope'}"
