"""The oracle and the CUDA path share nothing, and the product has no fallback.

Static checks (no GPU):
  * the package ``block_causal_linear_rope_b200`` (Python and CUDA sources) never
    imports or includes anything from ``oracle/``, and ``libblin.so`` neither
    links the oracle's library nor defines or calls one of its symbols;
  * ``oracle/`` never imports the package, the seeded input module or any of
    the CUDA sources; its C file includes only the C and OpenMP headers;
  * ``workloads/`` (the seeded inputs both sides draw from) imports neither;
  * ``bench.py`` imports the oracle only inside its CPU-baseline timers;
  * importing the package without its built library raises ImportError.
"""
import ast
import os
import re
import shutil
import subprocess
import sys

import pytest

import block_causal_linear_rope_b200 as blin

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "block_causal_linear_rope_b200")
ORACLE = os.path.join(ROOT, "oracle")
WORKLOADS = os.path.join(ROOT, "workloads")


def py_files(folder):
    for base, _, names in os.walk(folder):
        for n in sorted(names):
            if n.endswith(".py"):
                yield os.path.join(base, n)


def imported_modules(path):
    """Top-level module names a Python file imports, wherever the import sits."""
    tree = ast.parse(open(path).read(), path)
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            out.add(node.module.split(".")[0])
    return out


def includes(path):
    return re.findall(r'^\s*#\s*include\s*[<"]([^>"]+)[>"]', open(path).read(), flags=re.M)


def test_package_never_reaches_the_oracle():
    for f in py_files(PKG):
        assert not imported_modules(f) & {"oracle", "workloads"}, f
    csrc = os.path.join(PKG, "csrc")
    for n in sorted(os.listdir(csrc)):
        if n.endswith((".cu", ".cuh", ".h")):
            for inc in includes(os.path.join(csrc, n)):
                assert "oracle" not in inc, (n, inc)


def test_library_links_and_names_no_oracle_symbol():
    needed = subprocess.run(["readelf", "-d", blin.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in needed
    syms = subprocess.run(["nm", "-D", blin.LIB_PATH], capture_output=True, text=True).stdout
    assert syms and "blin_oracle" not in syms


def test_oracle_never_reaches_the_product():
    for f in py_files(ORACLE):
        assert not imported_modules(f) & {"block_causal_linear_rope_b200", "workloads", "torch"}, f
    c_files = [n for n in os.listdir(ORACLE) if n.endswith((".c", ".h"))]
    assert c_files
    for n in c_files:
        for inc in includes(os.path.join(ORACLE, n)):
            assert inc in {"math.h", "stdlib.h", "string.h", "stdint.h", "stddef.h", "omp.h"}, (n, inc)


def test_input_module_imports_neither_side():
    for f in py_files(WORKLOADS):
        assert not imported_modules(f) & {"block_causal_linear_rope_b200", "oracle"}, f


def test_bench_imports_the_oracle_only_in_its_cpu_timers():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), path)
    assert "oracle" not in {a.name for n in tree.body if isinstance(n, ast.Import) for a in n.names}
    owners = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for node in ast.walk(fn):
                if isinstance(node, ast.Import) and any(a.name == "oracle" for a in node.names):
                    owners.add(fn.name)
    assert owners == {"oracle_sample", "oracle_recurrence_rate"}


def test_package_without_its_library_refuses_to_import(tmp_path):
    pkg = tmp_path / "block_causal_linear_rope_b200"
    pkg.mkdir()
    shutil.copy(os.path.join(PKG, "__init__.py"), pkg / "__init__.py")
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n    import block_causal_linear_rope_b200\nexcept ImportError as e:\n"
            "    print('refused:', e); sys.exit(0)\n"
            "sys.exit(3)\n")
    r = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, cwd=str(tmp_path),
                       timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "libblin.so" in r.stdout and "missing" in r.stdout
