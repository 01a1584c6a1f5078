"""The oracle and the CUDA path share no code, and the product has no
fallback: static checks of the imports on both sides, and the binding's
import failing loudly without its library."""
import ast
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "activation_kv_sparsity_b200"


def _imports(path):
    tree = ast.parse(open(path).read())
    out = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            out.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            out.add(node.module.split(".")[0])
    return out


def _py_files(d):
    for base, _, files in os.walk(os.path.join(ROOT, d)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_oracle_imports_neither_the_library_nor_the_tests():
    for f in _py_files("oracle"):
        assert not _imports(f) & {PKG, "tests", "parity", "bench"}, f


def test_library_and_input_generator_never_import_the_oracle():
    for d in (PKG, "synth"):
        for f in _py_files(d):
            assert not _imports(f) & {"oracle", "tests", "parity"}, f
    for base, _, files in os.walk(os.path.join(ROOT, PKG, "csrc")):
        for f in files:
            text = open(os.path.join(base, f), errors="replace").read()
            assert "oracle" not in text, f


def test_binding_import_fails_without_the_library(tmp_path):
    pkg = tmp_path / PKG
    pkg.mkdir()
    shutil.copy(os.path.join(ROOT, PKG, "__init__.py"), pkg / "__init__.py")
    r = subprocess.run([sys.executable, "-c", f"import {PKG}"], cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0
    assert "libbytecross.so is missing" in r.stderr
