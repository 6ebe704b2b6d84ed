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


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("d", [32, 96, 4096])
def test_pack_fast_path_code_on_cpu_matches_oracle(tmp_path, bits, d):
    """The per-chunk code of the GPU pack fast path (pack32.cuh, the same functions the kernel
    calls), compiled for the host and run over every chunk, packs like the oracle, bit for bit."""
    import numpy as np
    from oracle import pack as pk
    exe = tmp_path / "pack32_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror", "-Wno-unknown-pragmas",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "pack32_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    n = 7
    codes = np.random.default_rng(bits * 100 + d).integers(0, 2 ** bits, (n, d), dtype=np.uint8)
    codes[0] = 2 ** bits - 1                  # all bits set: straddling fields must not collide
    (tmp_path / "codes.bin").write_bytes(codes.tobytes())
    r = subprocess.run([str(exe), str(bits), str(n), str(d), str(tmp_path / "codes.bin"),
                        str(tmp_path / "words.bin")], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    words = np.frombuffer((tmp_path / "words.bin").read_bytes(), np.uint32).reshape(n, -1)
    np.testing.assert_array_equal(words, pk.pack_rows(codes, bits))
