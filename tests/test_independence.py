"""The CUDA path and the oracle share no code, and the product path never reaches the oracle.

Static checks over the sources (no GPU): the package and its CUDA sources neither import, include nor load
anything under oracle/; the oracle imports nothing from the package (the seeded input generators in
weight_only_bit_route_b200/synthetic.py are passed to both sides by the tests, and hold none of the method's
arithmetic); bench.py imports the oracle only inside its CPU-baseline and reference legs; and the binding refuses
to import without the built library instead of falling back to anything else.
"""
import ast
import os
import re
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "weight_only_bit_route_b200")


def _files(top, exts):
    for d, _, fs in os.walk(top):
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def _imports(path):
    tree = ast.parse(open(path).read(), path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield node, a.name
        elif isinstance(node, ast.ImportFrom):
            yield node, (node.module or "")


def test_package_never_reaches_the_oracle():
    for path in _files(PKG, (".py",)):
        for _, name in _imports(path):
            assert name.split(".")[0] != "oracle", f"{path} imports {name}"
    for path in _files(PKG, (".cu", ".cuh", ".h", ".py")):
        src = open(path).read()
        assert not re.search(r"#include\s*[<\"][^>\"]*oracle", src), f"{path} includes an oracle header"
        assert "liboracle" not in src and "moe_oracle" not in src, f"{path} names the oracle's library or source"


def test_oracle_never_reaches_the_package():
    for path in _files(os.path.join(ROOT, "oracle"), (".py",)):
        for _, name in _imports(path):
            assert not name.startswith("weight_only_bit_route_b200"), f"{path} imports {name}"
    for path in _files(os.path.join(ROOT, "oracle"), (".c", ".h")):
        src = open(path).read()
        for inc in re.findall(r"#include\s*[<\"]([^>\"]+)[>\"]", src):
            assert inc in ("math.h", "stdint.h", "stdlib.h", "string.h", "omp.h"), f"{path} includes {inc}"


def test_synthetic_loads_neither_side():
    """The shared input module draws seeded numbers (numpy generators; torch only for the bf16 cast of what
    was drawn): it imports neither the binding, the expert-parallel module nor the oracle, and loads no library."""
    path = os.path.join(PKG, "synthetic.py")
    for _, name in _imports(path):
        assert name.split(".")[0] in ("dataclasses", "numpy", "torch", "math", "typing", "__future__"), name
    src = open(path).read()
    assert "ctypes" not in src and "CDLL" not in src


def test_bench_imports_the_oracle_only_in_its_cpu_legs():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), path)
    allowed = {"cpu_baseline", "run_reference"}
    for node in tree.body:
        if isinstance(node, (ast.Import, ast.ImportFrom)):
            names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
            assert all(n.split(".")[0] != "oracle" for n in names), "bench.py imports the oracle at module level"
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            if isinstance(node, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in node.names):
                assert fn.name in allowed, f"bench.py imports the oracle in {fn.name}"


def test_binding_refuses_to_import_without_the_library(tmp_path):
    """A copy of the package without libmoe.so cannot be imported: there is no fallback."""
    dst = tmp_path / "weight_only_bit_route_b200"
    dst.mkdir()
    for f in ("__init__.py", "moe.py", "synthetic.py"):
        src = os.path.join(PKG, f)
        if os.path.exists(src):
            (dst / f).write_text(open(src).read())
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n    import weight_only_bit_route_b200.moe\nexcept ImportError as e:\n    print('refused:', e)\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert "refused:" in r.stdout and "libmoe.so" in r.stdout, r.stdout
