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


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("n,d,ldw", [(5, 128, 128), (3, 1152, 1200), (70000, 128, 130)])
def test_w_gather_code_on_cpu(tmp_path, dtype, n, d, ldw):
    """The per-thread code of the sweep's W gather (gather4.cuh, the functions gather_w_kernel
    calls), run on the CPU over the host's launch grid (including more rows than grid.y), gives
    W[:, perm] widened to fp32 with the dead columns zeroed."""
    import numpy as np
    import torch
    exe = tmp_path / "gather4_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror", "-Wno-unknown-pragmas",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "gather4_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    rng = np.random.default_rng(n + d)
    W = torch.from_numpy(rng.standard_normal((n, ldw)).astype(np.float32))
    if dtype == "bf16":
        W = W.to(torch.bfloat16)
        raw = W.view(torch.int16).numpy().tobytes()
    else:
        raw = W.numpy().tobytes()
    perm = rng.permutation(d).astype(np.int32)
    dead = (rng.random(d) < 0.1).astype(np.uint8)
    for name, data in (("w.bin", raw), ("perm.bin", perm.tobytes()), ("dead.bin", dead.tobytes())):
        (tmp_path / name).write_bytes(data)
    r = subprocess.run([str(exe), dtype, str(n), str(d), str(ldw)] +
                       [str(tmp_path / x) for x in ("w.bin", "perm.bin", "dead.bin", "out.bin")],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.frombuffer((tmp_path / "out.bin").read_bytes(), np.float32).reshape(n, d)
    want = W.float().numpy()[:, :d][:, perm].copy()
    want[:, dead.astype(bool)] = 0.0
    np.testing.assert_array_equal(got, want)


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("part,d,ld,grid", [(0, 1, 1, 1), (0, 37, 37, 37), (0, 1500, 1500, 1184),
                                            (0, 1501, 1501, 3), (1, 37, 40, 37),
                                            (1, 1500, 1504, 1184), (1, 999, 1003, 7)])
def test_triangle_clear_index_math_on_cpu(tmp_path, part, d, ld, grid):
    """The triangle-clearing kernels' index arithmetic (tri_fill.cuh: row spans, a scalar head
    to a 16-byte boundary, 16-byte body, scalar tail) over a launch grid of whole rows per block
    clears exactly the strictly lower triangle (part 0) or the upper triangle with the diagonal
    (part 1, padded rows left alone) and nothing else, for rows of any alignment."""
    import numpy as np
    exe = tmp_path / "tri_fill_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "tri_fill_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe), str(part), str(d), str(ld), str(grid)], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.array([[c == "1" for c in line] for line in r.stdout.split()], dtype=bool)
    want = np.ones((d, ld), bool)
    rows, cols = np.indices((d, d))
    cleared = rows > cols if part == 0 else rows <= cols
    want[:, :d][cleared] = False
    np.testing.assert_array_equal(got, want)


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("d", [1, 37, 1100])
def test_permute_sym_index_math_on_cpu(tmp_path, d):
    """The act-order permutation of H (permute_sym_kernel's loops over the host's launch grid,
    tri_fill.cuh) writes exactly Hp[a][b] = H[pi a][pi b] on the upper triangle, reading only
    H's upper triangle, and nothing below the diagonal."""
    import numpy as np
    exe = tmp_path / "permute_sym_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "permute_sym_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    rng = np.random.default_rng(d)
    S = rng.standard_normal((d, d)).astype(np.float32)
    S = S + S.T
    H = np.triu(S) + np.tril(np.full((d, d), np.nan, np.float32), -1)   # lower part never read
    perm = rng.permutation(d).astype(np.int32)
    (tmp_path / "h.bin").write_bytes(H.tobytes())
    (tmp_path / "perm.bin").write_bytes(perm.tobytes())
    r = subprocess.run([str(exe), str(d), str(tmp_path / "h.bin"), str(tmp_path / "perm.bin"),
                        str(tmp_path / "out.bin")], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.frombuffer((tmp_path / "out.bin").read_bytes(), np.float32).reshape(d, d)
    iu = np.triu_indices(d)
    np.testing.assert_array_equal(got[iu], S[perm][:, perm][iu])
    assert np.all(got[np.tril_indices(d, -1)] == -1.0)


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("n,d", [(3, 128), (70000, 256), (5, 4096)])
def test_unpermute_codes_index_math_on_cpu(tmp_path, n, d):
    """unpermute_codes_kernel's loops over the host's launch grid (more rows than grid y
    included) put every sweep-order code back at its original column: codes[:, perm] = cs."""
    import numpy as np
    exe = tmp_path / "unpermute_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "unpermute_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    rng = np.random.default_rng(n + d)
    cs = rng.integers(0, 16, (n, d), dtype=np.uint8)
    perm = rng.permutation(d).astype(np.int32)
    (tmp_path / "cs.bin").write_bytes(cs.tobytes())
    (tmp_path / "perm.bin").write_bytes(perm.tobytes())
    r = subprocess.run([str(exe), str(n), str(d), str(tmp_path / "cs.bin"),
                        str(tmp_path / "perm.bin"), str(tmp_path / "out.bin")],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.frombuffer((tmp_path / "out.bin").read_bytes(), np.uint8).reshape(n, d)
    want = np.empty_like(cs)
    want[:, perm] = cs
    np.testing.assert_array_equal(got, want)


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc")
def test_wait_timeout_check_kernel_builds(tmp_path):
    """The test-only bounded-wait kernel (run by tests/test_gpu_failure.py) cross-compiles for
    sm_100a against the library's own wait helpers."""
    so = tmp_path / "wait_timeout_check.so"
    r = subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                        "-Xcompiler", "-fPIC", "-I",
                        os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "wait_timeout_check.cu"), "-o", str(so),
                        "-lcuda"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("n_tb,grp,n_split", [(1, 1, 1), (16, 16, 32), (16, 12, 3), (112, 12, 16),
                                              (7, 3, 2), (5, 8, 1)])
def test_syrk_unit_order_on_cpu(tmp_path, n_tb, grp, n_split):
    """The SYRK's work units (syrk_units.cuh, the kernel's own mapping) cover every upper tile
    (ib <= jb) in every token range exactly once, and inside a group run range by range."""
    import numpy as np
    exe = tmp_path / "syrk_units_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "syrk_units_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe), str(n_tb), str(grp), str(n_split)], capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    got = np.array([list(map(int, line.split())) for line in r.stdout.splitlines()])
    want = {(i, j, s) for j in range(n_tb) for i in range(j + 1) for s in range(n_split)}
    assert len(got) == len(want) and {tuple(x) for x in got} == want
    # consecutive units of one group share the token range until the group's tiles are done
    grp_id = (got[:, 0] // grp) * 100000 + (got[:, 1] // grp)
    for g in np.unique(grp_id):
        splits = got[grp_id == g, 2]
        assert np.all(np.diff(splits) >= 0)


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_gemv_pair_decoding_on_cpu(tmp_path, bits):
    """The tensor-core GEMV's pair decoding (gemv_pairs.cuh, the functions the kernel calls):
    every code of a 32-code run, packed by the oracle, comes back once, as a clean in-place field
    of an fp16 half, at the run column the activation pairing assumes."""
    import numpy as np
    from oracle import pack as pk
    exe = tmp_path / "gemv_pairs_check"
    r = subprocess.run(["g++", "-std=c++17", "-O2", "-Wall", "-Werror", "-Wno-unknown-pragmas",
                        "-I", os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                        os.path.join(ROOT, "tests", "c", "gemv_pairs_check.cpp"), "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    n = 300
    codes = np.random.default_rng(bits).integers(0, 2 ** bits, (n, 32), dtype=np.uint8)
    codes[0] = 2 ** bits - 1
    codes[1] = 0
    words = pk.pack_rows(codes, bits)               # oracle packing: `bits` words per 32 codes
    (tmp_path / "in.bin").write_bytes(words.astype(np.uint32).tobytes())
    r = subprocess.run([str(exe), str(bits), str(n), str(tmp_path / "in.bin"),
                        str(tmp_path / "out.bin")], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.returncode
    out = np.frombuffer((tmp_path / "out.bin").read_bytes(), np.uint8).reshape(n, 32)
    np.testing.assert_array_equal(out, codes)
