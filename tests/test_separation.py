"""The separation the parity claims rest on, checked on the sources:

* the library package (the product path) imports neither the oracle nor the
  seeded-input module, and its C/CUDA sources include nothing from them;
* the oracle imports neither the library nor the seeded-input module, and
  the seeded-input module imports neither the oracle nor the library;
* bench.py reaches the oracle only inside its CPU-baseline timing function;
* without its shared library the package raises instead of computing.
"""
import ast
import glob
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "expert_offloaded_serving_b200"


def top_modules(path):
    """Top-level names of every module a Python file imports (absolute imports)."""
    tree = ast.parse(open(path).read())
    out = set()
    for n in ast.walk(tree):
        if isinstance(n, ast.Import):
            out |= {a.name.split(".")[0] for a in n.names}
        elif isinstance(n, ast.ImportFrom) and n.level == 0 and n.module:
            out.add(n.module.split(".")[0])
    return out


def files(sub):
    return sorted(glob.glob(os.path.join(ROOT, sub, "*.py")))


def test_product_package_imports_neither_oracle_nor_inputs():
    for f in files(PKG):
        assert not top_modules(f) & {"oracle", "synth"}, f
    for f in glob.glob(os.path.join(ROOT, PKG, "csrc", "*")) + glob.glob(os.path.join(ROOT, "include", "*")):
        text = open(f, errors="replace").read()
        assert "oracle/" not in text and "synth/" not in text, f


def test_oracle_and_inputs_import_neither_each_other_nor_the_library():
    for f in files("oracle"):
        assert not top_modules(f) & {PKG, "synth", "torch"}, f
    for f in files("synth"):
        assert not top_modules(f) & {PKG, "oracle"}, f


def test_bench_reaches_the_oracle_only_in_its_cpu_baseline_timing():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py")).read())
    users = set()
    for fn in ast.walk(tree):
        if isinstance(fn, ast.FunctionDef):
            for n in ast.walk(fn):
                if isinstance(n, ast.ImportFrom) and n.module and n.module.split(".")[0] == "oracle":
                    users.add(fn.name)
                if isinstance(n, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in n.names):
                    users.add(fn.name)
    top = {n.module.split(".")[0] for n in tree.body if isinstance(n, ast.ImportFrom) and n.module}
    top |= {a.name.split(".")[0] for n in tree.body if isinstance(n, ast.Import) for a in n.names}
    assert "oracle" not in top
    assert users == {"oracle_layer_times"}


def test_package_without_its_library_raises():
    """With its shared library missing, the package's first call raises
    instead of falling back to anything."""
    code = (f"import sys; sys.path.insert(0, {ROOT!r}); import {PKG} as ft\n"
            f"ft.LIB_PATH = {os.path.join(ROOT, PKG, 'no_such_lib.so')!r}\n"
            "try:\n    ft.ft_blob_stride(256, 128)\nexcept RuntimeError as e:\n    print('raised:', e)\n"
            "else:\n    print('computed')\n")
    p = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert "raised:" in p.stdout and "missing" in p.stdout, p.stdout + p.stderr
