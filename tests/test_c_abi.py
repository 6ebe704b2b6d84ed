"""The boundary is a plain C ABI: a C99 program compiled against include/gptq.h alone links the
library and gets the documented host-side results (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_client_compiles_links_and_runs(tmp_path):
    import post_weight_quantization_18_b200 as G
    libdir = os.path.dirname(G.LIB_PATH)
    exe = tmp_path / "gptq_abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "gptq_abi_check.c"), "-o", str(exe),
           "-L", libdir, "-l:" + os.path.basename(G.LIB_PATH), "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
