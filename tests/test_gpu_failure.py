"""Failure detection on the GPU, without a GPU fault.

* A status word that already holds an error makes every later call that is given it do no work
  (include/gptq.h, conventions): sentinel-filled outputs stay untouched.
* A bounded wait that nothing completes gives up after its limit, records GPTQ_ERR_TIMEOUT and
  returns, and the context stays usable: a test-only kernel built from the library's own
  wait helpers (tests/c/wait_timeout_check.cu) waits 1 ms on an mbarrier that no thread arrives
  on and no copy completes (no asynchronous copy is in flight).
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from gpu_util import make_inputs

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ERR_NOT_SPD, ERR_TIMEOUT = 16, 18


def test_preset_status_skips_all_work():
    import post_weight_quantization_18_b200 as G
    n, d, N = 64, 256, 2048
    W, X = make_inputs(n, d, N, seed=11)
    Xd, Wd = X.cuda(), W.cuda()
    st = torch.tensor([ERR_NOT_SPD, 7], dtype=torch.int32, device="cuda")
    p = G.make_params(4, 128, order=G.GPTQ_ORDER_DESC_ACT)
    H = torch.full((d, d), 3.0, device="cuda")
    U = torch.full((d, d), 5.0, device="cuda")
    perm = torch.full((d,), -3, dtype=torch.int32, device="cuda")
    dead = torch.full((d,), 9, dtype=torch.uint8, device="cuda")
    G.gptq_hessian_accumulate(H, Xd, 2.0, False, st)
    G.gptq_hessian_accumulate(H, Xd, 2.0, True, st)
    G.gptq_prepare_hinv(H, p, U, perm, dead, None, st)
    codes = torch.full((n, d), 200, dtype=torch.uint8, device="cuda")
    S = torch.full((n, 2), -1.0, device="cuda")
    Z = torch.full((n, 2), -2.0, device="cuda")
    gi = torch.full((d,), -5, dtype=torch.int32, device="cuda")
    ws = torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device="cuda")
    Ug = torch.eye(d, device="cuda")
    pg = torch.arange(d, dtype=torch.int32, device="cuda")
    dg = torch.zeros(d, dtype=torch.uint8, device="cuda")
    G.gptq_quantize_layer(Wd, Ug, pg, dg, p, codes, S, Z, gi, ws, st)
    G.gptq_quantize_layer_noalloc(Wd, Ug, pg, dg, p, codes, S, Z, gi, st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [ERR_NOT_SPD, 7]
    assert torch.all(H == 3.0) and torch.all(U == 5.0)
    assert torch.all(perm == -3) and torch.all(dead == 9)
    assert torch.all(codes == 200) and torch.all(S == -1.0) and torch.all(Z == -2.0)
    assert torch.all(gi == -5)
    # The same calls with a clear status word do their work.
    st.zero_()
    out = G.quantize_layer(Wd, X=Xd, bits=4, group_size=128)
    torch.cuda.synchronize()
    assert out.codes.max().item() <= 15


def _build_wait_check(tmp_path):
    so = tmp_path / "wait_timeout_check.so"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-shared",
                    "-Xcompiler", "-fPIC", "-I",
                    os.path.join(ROOT, "post_weight_quantization_18_b200", "csrc"),
                    os.path.join(ROOT, "tests", "c", "wait_timeout_check.cu"), "-o", str(so),
                    "-lcuda"], check=True)
    lib = ctypes.CDLL(str(so))
    lib.wait_nobody.argtypes = [ctypes.c_void_p, ctypes.c_ulonglong, ctypes.c_void_p,
                                ctypes.c_void_p]
    lib.wait_nobody.restype = ctypes.c_int
    return lib


def test_bounded_wait_times_out_and_reports(tmp_path):
    lib = _build_wait_check(tmp_path)
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    res = torch.zeros(3, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.wait_nobody(st.data_ptr(), 1_000_000, res.data_ptr(), stream) == 0
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [ERR_TIMEOUT, 99]
    assert res.cpu().tolist() == [1, 0, 1]
    # The context is still usable: the library runs a layer and agrees with itself.
    import post_weight_quantization_18_b200 as G
    W, X = make_inputs(32, 128, 1024, seed=12)
    a = G.quantize_layer(W.cuda(), X=X.cuda(), bits=4, group_size=128)
    b = G.quantize_layer(W.cuda(), X=X.cuda(), bits=4, group_size=128)
    torch.cuda.synchronize()
    assert np.array_equal(a.codes.cpu().numpy(), b.codes.cpu().numpy())
