"""The product path has no CPU fallback and never reaches the oracle.

* A copy of the package without the built library refuses to import (ImportError that says so),
  instead of falling back to anything else.
* No module of the package imports the oracle (it is test infrastructure only).
"""
import ast
import os
import shutil
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "post_weight_quantization_18_b200")


def test_package_without_library_refuses_to_import(tmp_path):
    dst = tmp_path / "post_weight_quantization_18_b200"
    dst.mkdir()
    for name in os.listdir(PKG):
        if name.endswith(".py"):
            shutil.copy(os.path.join(PKG, name), dst / name)
    r = subprocess.run([sys.executable, "-c", "import post_weight_quantization_18_b200"],
                       cwd=tmp_path, capture_output=True, text=True, timeout=300,
                       env={**os.environ, "PYTHONPATH": str(tmp_path)})
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "no CPU fallback" in r.stderr, r.stderr[-2000:]


def test_package_never_imports_the_oracle():
    for name in os.listdir(PKG):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(PKG, name)).read())
        for node in ast.walk(tree):
            mods = []
            if isinstance(node, ast.Import):
                mods = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom) and node.module:
                mods = [node.module]
            assert not any(m == "oracle" or m.startswith("oracle.") for m in mods), (name, mods)
