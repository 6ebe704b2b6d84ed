"""The C ABI library loads, exports every function include/gptq.h declares, and rejects bad
arguments on the host before touching the GPU (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    path = __graft_entry__._build_module().build()
    return ctypes.CDLL(path)


def declared_functions():
    src = open(os.path.join(ROOT, "include", "gptq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*((?:gptq|rtn)_\w+)\s*\(", src,
                                 flags=re.M)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted([
        "gptq_dequant_gemm", "gptq_dequant_gemv", "gptq_gemm_f32", "gptq_hessian_accumulate",
        "gptq_pack",
        "gptq_prepare_hinv", "gptq_quantize_pack_layer",
        "gptq_quantize_layer", "gptq_quantize_layer_noalloc", "gptq_status_string",
        "gptq_workspace_size", "rtn_quantize"])


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_names_match_header():
    import post_weight_quantization_18_b200 as G
    assert sorted(G.EXPORTED) == declared_functions()
    for name in declared_functions():
        assert callable(getattr(G, name))


class P(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("sym", ctypes.c_int32),
                ("order", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("percdamp", ctypes.c_float), ("static_groups", ctypes.c_int32)]


def test_status_strings(lib):
    lib.gptq_status_string.restype = ctypes.c_char_p
    names = {c: lib.gptq_status_string(c).decode() for c in (0, 1, 2, 3, 4, 16, 17, 18, 99)}
    assert names[0] == "GPTQ_OK" and names[16] == "GPTQ_ERR_NOT_SPD"
    assert names[18] == "GPTQ_ERR_TIMEOUT" and names[99] == "GPTQ_ERR_UNKNOWN"


def test_workspace_size(lib):
    lib.gptq_workspace_size.restype = ctypes.c_size_t
    lib.gptq_workspace_size.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(P)]
    ok = P(4, 128, 0, 0, 128, 0.01)
    assert lib.gptq_workspace_size(4096, 4096, ctypes.byref(ok)) == 2 * 4096 * 4096 * 4
    act = P(3, 128, 0, 1, 128, 0.01)
    # a permuted order adds the sweep-order codes and the inverse permutation (int32 per column)
    assert lib.gptq_workspace_size(4096, 4096, ctypes.byref(act)) == \
        2 * 4096 * 4096 * 4 + 4096 * 4096 + 4096 * 4
    # static groups use the same inverse permutation
    st = P(4, 128, 0, 1, 128, 0.01, 1)
    assert lib.gptq_workspace_size(4096, 4096, ctypes.byref(st)) == \
        2 * 4096 * 4096 * 4 + 4096 * 4096 + 4096 * 4
    for bad in (P(5, 128, 0, 0, 128, 0.01), P(4, 96, 0, 0, 128, 0.01), P(4, 128, 0, 0, 64, 0.01),
                P(4, 128, 2, 0, 128, 0.01), P(4, 128, 0, 3, 128, 0.01), P(4, 6, 0, 0, 128, 0.01),
                P(4, 128, 0, 0, 128, -1.0), P(4, -1, 1, 0, 128, 0.01, 1),
                P(4, 128, 0, 1, 128, 0.01, 2)):
        assert lib.gptq_workspace_size(4096, 4096, ctypes.byref(bad)) == 0
    assert lib.gptq_workspace_size(0, 4096, ctypes.byref(ok)) == 0


def test_invalid_arguments_rejected_on_host(lib):
    V = ctypes.c_void_p
    fake = V(0x1000)  # never dereferenced: every call below fails its host-side checks
    lib.gptq_hessian_accumulate.argtypes = [V, ctypes.c_int64, ctypes.c_int64, V, ctypes.c_int,
                                            ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                            ctypes.c_int, V, V]
    assert lib.gptq_hessian_accumulate(None, 64, 64, fake, 0, 10, 64, 2.0, 0, None, None) == 1
    assert lib.gptq_hessian_accumulate(fake, 64, 32, fake, 0, 10, 64, 2.0, 0, None, None) == 1
    assert lib.gptq_hessian_accumulate(fake, 64, 64, fake, 0, 10, 32, 2.0, 0, None, None) == 1
    assert lib.gptq_hessian_accumulate(fake, 64, 64, fake, 7, 10, 64, 2.0, 0, None, None) == 2
    assert lib.gptq_hessian_accumulate(fake, 64, 64, fake, 0, 10, 66, 2.0, 0, None, None) == 1
    p = P(4, 128, 0, 0, 128, 0.01)
    lib.gptq_quantize_layer.argtypes = [V, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_int64, V, V, V, ctypes.POINTER(P), V, V, V, V, V,
                                        ctypes.c_size_t, V, V]
    args = lambda d_in, ws_bytes: (fake, 0, d_in, 16, d_in, fake, fake, fake, ctypes.byref(p), fake,
                                   fake, fake, fake, fake, ws_bytes, None, None)
    assert lib.gptq_quantize_layer(*args(100, 1 << 30)) == 1      # d_in not a multiple of 128
    assert lib.gptq_quantize_layer(*args(256, 16)) == 3           # workspace too small
    lib.gptq_pack.argtypes = [V, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, V, V,
                              ctypes.c_int64, V, V, V, V]
    assert lib.gptq_pack(fake, 4, 64, 5, fake, fake, 1, fake, fake, fake, None) == 1
    lib.rtn_quantize.argtypes = [V, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                 ctypes.POINTER(P), V, V, V, V]
    bad_g = P(4, 100, 0, 0, 128, 0.01)
    assert lib.rtn_quantize(fake, 0, 256, 4, 256, ctypes.byref(bad_g), fake, fake, fake, None) == 1
    lib.gptq_prepare_hinv.argtypes = [V, ctypes.c_int64, ctypes.POINTER(P), V, V, V, V,
                                      ctypes.c_size_t, V, V]
    assert lib.gptq_prepare_hinv(fake, 64, ctypes.byref(p), fake, None, fake, None, 0, None,
                                 None) == 1


def test_dequant_gemv_rejects_bad_arguments_on_host(lib):
    V, I64 = ctypes.c_void_p, ctypes.c_int64
    lib.gptq_dequant_gemv.argtypes = [V, I64, I64, ctypes.c_int, V, V, I64, ctypes.c_int, V, V,
                                      I64, I64, V, I64, V]
    fake = V(0x1000)  # 16-byte aligned, never dereferenced: every call fails its checks
    ok = (fake, 64, 128, 4, fake, fake, 1, 128, None, fake, 1, 128, fake, 64, None)

    def call(**kw):
        names = ["q", "n", "d", "bits", "s", "z", "G", "g", "gidx", "x", "b", "ldx", "y", "ldy",
                 "st"]
        args = dict(zip(names, ok))
        args.update(kw)
        return lib.gptq_dequant_gemv(*[args[k] for k in names])

    assert call(q=None) == 1
    assert call(d=100) == 1                 # d_in not a multiple of 32
    assert call(bits=5) == 1
    assert call(b=0) == 1 and call(b=9) == 1
    assert call(ldx=132) == 1               # not a multiple of 8
    assert call(ldy=10) == 1
    assert call(x=V(0x1004)) == 1           # X not 16-byte aligned
    assert call(g=48) == 1                  # group size does not divide d_in
    assert call(G=2) == 1                   # n_groups disagrees with group_size
    assert call(g=-1, G=2) == 1


def test_dequant_gemm_rejects_bad_arguments_on_host(lib):
    V, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.gptq_dequant_gemm.argtypes = [V, I64, I64, V, V, I64, I, V, I64, I64, V, I64, V, V]
    lib.gptq_dequant_gemm.restype = I
    fake = V(0x1000)  # 16-byte aligned, never dereferenced: every call fails its checks
    ok = dict(q=fake, n=64, d=256, s=fake, z=fake, G=2, g=128, x=fake, m=40, ldx=256, y=fake,
              ldy=64, st=None, stream=None)
    names = list(ok)

    def call(**kw):
        args = dict(ok)
        args.update(kw)
        return lib.gptq_dequant_gemm(*[args[k] for k in names])

    assert call(q=None) == 1 and call(x=None) == 1 and call(y=None) == 1
    assert call(d=192, G=1, g=-1) == 1      # d_in not a multiple of 128
    assert call(m=0) == 1
    assert call(ldx=260) == 1               # not a multiple of 8
    assert call(ldy=63) == 1
    assert call(x=V(0x1004)) == 1           # X not 16-byte aligned
    assert call(g=64, G=4) == 1             # groups must be whole multiples of 128 columns
    assert call(G=3) == 1                   # n_groups disagrees with group_size
    assert call(g=-1, G=2) == 1


def test_gemm_host_checks(lib):
    """gptq_gemm_f32 rejects null pointers, impossible shapes and short leading dimensions on
    the host (nothing is launched; the fake pointers are never dereferenced)."""
    V, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.gptq_gemm_f32.argtypes = [I64, I64, I64, ctypes.c_float, V, I64, I, V, I64, I,
                                  ctypes.c_float, V, I64, V, V]
    lib.gptq_gemm_f32.restype = I
    f = 0x1000

    def call(M=8, N=8, K=8, A=f, lda=8, ta=0, B=f, ldb=8, tb=0, C=f, ldc=8):
        return lib.gptq_gemm_f32(M, N, K, 1.0, A, lda, ta, B, ldb, tb, 0.0, C, ldc, None, None)
    assert call(C=None) == 1
    assert call(A=None) == 1 and call(B=None) == 1
    assert call(M=0) == 1 and call(N=0) == 1 and call(K=-1) == 1
    assert call(lda=7) == 1 and call(ldb=7) == 1 and call(ldc=7) == 1
    assert call(ta=1, lda=7, M=8, K=9) == 1          # op(A)^T rows are M long
    assert call(ta=2) == 1 and call(tb=2) == 1
    assert call(C=0x1002) == 1                        # misaligned fp32 pointer
