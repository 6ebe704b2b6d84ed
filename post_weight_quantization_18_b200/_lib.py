"""ctypes binding of libgptq_b200.so — argument marshalling only.

Every function here has the name of the C entry point it calls (include/gptq.h), takes torch
CUDA tensors, checks shapes/dtypes/devices on the host, passes raw pointers and the current CUDA
stream, and raises GPTQError on a non-OK return. No arithmetic of the method happens here.
There is no fallback: if the shared library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgptq_b200.so")

GPTQ_OK = 0
GPTQ_ERR_INVALID_ARG = 1
GPTQ_ERR_UNSUPPORTED = 2
GPTQ_ERR_WORKSPACE = 3
GPTQ_ERR_CUDA = 4
GPTQ_ERR_NOT_SPD = 16
GPTQ_ERR_NONFINITE = 17
GPTQ_ERR_TIMEOUT = 18

GPTQ_BF16 = 0
GPTQ_F32 = 1
GPTQ_ORDER_NATURAL = 0
GPTQ_ORDER_DESC_ACT = 1
GPTQ_ORDER_GIVEN = 2

EXPORTED = ("gptq_workspace_size", "gptq_hessian_accumulate", "gptq_prepare_hinv",
            "gptq_quantize_layer", "gptq_pack", "rtn_quantize", "gptq_status_string",
            "gptq_quantize_layer_noalloc", "gptq_dequant_gemv", "gptq_gemm_f32",
            "gptq_quantize_pack_layer", "gptq_dequant_gemm")
GPTQ_NOALLOC_SCRATCH_BYTES = 32 << 20


class GPTQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


class gptq_params(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("sym", ctypes.c_int32),
                ("order", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("percdamp", ctypes.c_float), ("static_groups", ctypes.c_int32)]


def make_params(bits: int = 4, group_size: int = 128, sym: bool = False, order: int = 0,
                block_size: int = 128, percdamp: float = 0.01,
                static_groups: bool = False) -> gptq_params:
    return gptq_params(int(bits), int(group_size), int(bool(sym)), int(order), int(block_size),
                       float(percdamp), int(bool(static_groups)))


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python post_weight_quantization_18_b200/build.py`"
            " (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I64, I32, F32, SZ = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float,
                            ctypes.c_size_t)
    PP = ctypes.POINTER(gptq_params)
    lib.gptq_workspace_size.argtypes = [I64, I64, PP]
    lib.gptq_workspace_size.restype = SZ
    lib.gptq_hessian_accumulate.argtypes = [P, I64, I64, P, I32, I64, I64, F32, I32, P, P]
    lib.gptq_hessian_accumulate.restype = I32
    lib.gptq_prepare_hinv.argtypes = [P, I64, PP, P, P, P, P, SZ, P, P]
    lib.gptq_prepare_hinv.restype = I32
    lib.gptq_quantize_layer.argtypes = [P, I32, I64, I64, I64, P, P, P, PP, P, P, P, P, P, SZ, P, P]
    lib.gptq_quantize_layer.restype = I32
    lib.gptq_quantize_layer_noalloc.argtypes = [P, I32, I64, I64, I64, P, P, P, PP, P, P, P, P,
                                                P, P]
    lib.gptq_quantize_layer_noalloc.restype = I32
    lib.gptq_pack.argtypes = [P, I64, I64, I32, P, P, I64, P, P, P, P]
    lib.gptq_pack.restype = I32
    lib.rtn_quantize.argtypes = [P, I32, I64, I64, I64, PP, P, P, P, P]
    lib.rtn_quantize.restype = I32
    lib.gptq_dequant_gemv.argtypes = [P, I64, I64, I32, P, P, I64, I32, P, P, I64, I64, P, I64, P]
    lib.gptq_dequant_gemv.restype = I32
    lib.gptq_dequant_gemm.argtypes = [P, I64, I64, P, P, I64, I32, P, I64, I64, P, I64, P, P]
    lib.gptq_dequant_gemm.restype = I32
    lib.gptq_gemm_f32.argtypes = [I64, I64, I64, F32, P, I64, I32, P, I64, I32, F32, P, I64, P, P]
    lib.gptq_gemm_f32.restype = I32
    lib.gptq_quantize_pack_layer.argtypes = [P, I32, I64, I64, I64, P, P, P, PP, P, P, P, P, P, P,
                                             P, SZ, P, P]
    lib.gptq_quantize_pack_layer.restype = I32
    lib.gptq_status_string.argtypes = [I32]
    lib.gptq_status_string.restype = ctypes.c_char_p
    return lib


_lib = _load()


def gptq_status_string(code: int) -> str:
    return _lib.gptq_status_string(int(code)).decode()


status_string = gptq_status_string


def _check(rc: int, where: str) -> None:
    if rc != GPTQ_OK:
        raise GPTQError(rc, where)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, name: str, dtype=None, ndim=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


def _row_major(t: torch.Tensor, name: str) -> None:
    if t.dim() == 2 and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit stride along its last dim")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GPTQ_BF16
    if t.dtype == torch.float32:
        return GPTQ_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def gptq_workspace_size(d_out: int, d_in: int, params: gptq_params) -> int:
    return int(_lib.gptq_workspace_size(int(d_out), int(d_in), ctypes.byref(params)))


def gptq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor, alpha: float = 2.0,
                            accumulate: bool = False, dev_status: torch.Tensor | None = None
                            ) -> None:
    """H[:d, :d] upper (+)= alpha * X^T X for token-major X [n_tokens, d]."""
    _dev(H, "H", torch.float32, 2)
    _dev(X, "X", None, 2)
    _row_major(H, "H")
    _row_major(X, "X")
    d = X.shape[1]
    if H.shape[0] < d or H.shape[1] < d:
        raise ValueError("H is smaller than d_in x d_in")
    rc = _lib.gptq_hessian_accumulate(_ptr(H), d, H.stride(0), _ptr(X), _dtype_code(X),
                                      X.shape[0], X.stride(0), float(alpha), int(bool(accumulate)),
                                      _ptr(dev_status), _stream())
    _check(rc, "gptq_hessian_accumulate")


def gptq_prepare_hinv(H: torch.Tensor, params: gptq_params, U: torch.Tensor, perm: torch.Tensor,
                      dead: torch.Tensor, ws: torch.Tensor | None = None,
                      dev_status: torch.Tensor | None = None) -> None:
    """H (clobbered) -> U upper Cholesky factor of H_damped^-1, perm, dead."""
    d = H.shape[0]
    _dev(H, "H", torch.float32, 2)
    _dev(U, "U", torch.float32, 2)
    _dev(perm, "perm", torch.int32, 1)
    _dev(dead, "dead", torch.uint8, 1)
    if H.shape != (d, d) or U.shape != (d, d) or not H.is_contiguous() or not U.is_contiguous():
        raise ValueError("H and U must be contiguous d x d")
    if perm.numel() != d or dead.numel() != d:
        raise ValueError("perm / dead must have d entries")
    rc = _lib.gptq_prepare_hinv(_ptr(H), d, ctypes.byref(params), _ptr(U), _ptr(perm), _ptr(dead),
                                _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                _ptr(dev_status), _stream())
    _check(rc, "gptq_prepare_hinv")


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor, dead: torch.Tensor,
                        params: gptq_params, codes: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor, g_idx: torch.Tensor, ws: torch.Tensor,
                        dev_status: torch.Tensor | None = None) -> None:
    """The column sweep of one layer (outputs written into the given tensors)."""
    _dev(W, "W", None, 2)
    _row_major(W, "W")
    n, d = W.shape
    _dev(U, "U", torch.float32, 2)
    _dev(codes, "codes", torch.uint8, 2)
    _dev(scales, "scales", torch.float32, 2)
    _dev(zeros, "zeros", torch.float32, 2)
    _dev(g_idx, "g_idx", torch.int32, 1)
    _dev(ws, "ws")
    G = 1 if params.group_size == -1 else d // params.group_size
    if codes.shape != (n, d) or not codes.is_contiguous():
        raise ValueError("codes must be contiguous [d_out, d_in]")
    if scales.shape != (n, G) or zeros.shape != (n, G) or not scales.is_contiguous() \
            or not zeros.is_contiguous():
        raise ValueError("scales / zeros must be contiguous [d_out, n_groups]")
    if U.shape != (d, d) or g_idx.numel() != d:
        raise ValueError("U must be d_in x d_in and g_idx must have d_in entries")
    rc = _lib.gptq_quantize_layer(_ptr(W), _dtype_code(W), W.stride(0), n, d, _ptr(U), _ptr(perm),
                                  _ptr(dead), ctypes.byref(params), _ptr(codes), _ptr(scales),
                                  _ptr(zeros), _ptr(g_idx), _ptr(ws),
                                  ws.numel() * ws.element_size(), _ptr(dev_status), _stream())
    _check(rc, "gptq_quantize_layer")


def gptq_quantize_layer_noalloc(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor,
                                dead: torch.Tensor, params: gptq_params, codes: torch.Tensor,
                                scales: torch.Tensor, zeros: torch.Tensor, g_idx: torch.Tensor,
                                dev_status: torch.Tensor | None = None) -> None:
    """gptq_quantize_layer with the library's own fixed scratch array instead of a caller buffer
    (for callers that cannot allocate device memory); layers whose scratch exceeds
    GPTQ_NOALLOC_SCRATCH_BYTES are rejected with GPTQ_ERR_WORKSPACE."""
    _dev(W, "W", None, 2)
    _row_major(W, "W")
    n, d = W.shape
    _dev(U, "U", torch.float32, 2)
    _dev(codes, "codes", torch.uint8, 2)
    _dev(scales, "scales", torch.float32, 2)
    _dev(zeros, "zeros", torch.float32, 2)
    _dev(g_idx, "g_idx", torch.int32, 1)
    G = 1 if params.group_size == -1 else d // params.group_size
    if codes.shape != (n, d) or not codes.is_contiguous():
        raise ValueError("codes must be contiguous [d_out, d_in]")
    if scales.shape != (n, G) or zeros.shape != (n, G) or not scales.is_contiguous() \
            or not zeros.is_contiguous():
        raise ValueError("scales / zeros must be contiguous [d_out, n_groups]")
    if U.shape != (d, d) or g_idx.numel() != d:
        raise ValueError("U must be d_in x d_in and g_idx must have d_in entries")
    rc = _lib.gptq_quantize_layer_noalloc(_ptr(W), _dtype_code(W), W.stride(0), n, d, _ptr(U),
                                          _ptr(perm), _ptr(dead), ctypes.byref(params),
                                          _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(g_idx),
                                          _ptr(dev_status), _stream())
    _check(rc, "gptq_quantize_layer_noalloc")


def gptq_pack(codes: torch.Tensor, bits: int, scales: torch.Tensor, zeros: torch.Tensor,
              qweight: torch.Tensor, scales_f16: torch.Tensor, zeros_f16: torch.Tensor) -> None:
    _dev(codes, "codes", torch.uint8, 2)
    n, d = codes.shape
    G = scales.shape[1]
    for t, nm, dt in ((qweight, "qweight", torch.int32), (scales_f16, "scales_f16", torch.int16),
                      (zeros_f16, "zeros_f16", torch.int16)):
        _dev(t, nm)
        if t.element_size() != (4 if dt == torch.int32 else 2) or not t.is_contiguous():
            raise ValueError(f"{nm} has the wrong element size or layout")
    if qweight.shape != (n, (d * bits + 31) // 32):
        raise ValueError("qweight must be [d_out, ceil(d_in*bits/32)]")
    if scales_f16.shape != (n, G) or zeros_f16.shape != (n, G) or zeros.shape != (n, G):
        raise ValueError("scales / zeros shapes disagree")
    rc = _lib.gptq_pack(_ptr(codes), n, d, int(bits), _ptr(scales), _ptr(zeros), G, _ptr(qweight),
                        _ptr(scales_f16), _ptr(zeros_f16), _stream())
    _check(rc, "gptq_pack")


def gptq_dequant_gemv(qweight: torch.Tensor, d_in: int, bits: int, scales_f16: torch.Tensor,
                      zeros_f16: torch.Tensor, group_size: int, g_idx: torch.Tensor | None,
                      X: torch.Tensor, Y: torch.Tensor) -> None:
    """Y [batch, d_out] (fp32) = X [batch, d_in] (fp16) @ W_hat^T from the packed layer."""
    for t, nm in ((qweight, "qweight"), (scales_f16, "scales_f16"), (zeros_f16, "zeros_f16"),
                  (X, "X"), (Y, "Y")):
        _dev(t, nm)
    if X.dtype != torch.float16 or Y.dtype != torch.float32:
        raise ValueError("X must be float16 and Y float32")
    if g_idx is not None:
        _dev(g_idx, "g_idx", torch.int32, 1)
    X2 = X.reshape(-1, X.shape[-1])
    Y2 = Y.reshape(-1, Y.shape[-1])
    _row_major(X2, "X")
    _row_major(Y2, "Y")
    n = qweight.shape[0]
    rc = _lib.gptq_dequant_gemv(_ptr(qweight), n, int(d_in), int(bits), _ptr(scales_f16),
                                _ptr(zeros_f16), scales_f16.shape[1], int(group_size), _ptr(g_idx),
                                _ptr(X2), X2.shape[0], X2.stride(0), _ptr(Y2), Y2.stride(0),
                                _stream())
    _check(rc, "gptq_dequant_gemv")


def gptq_dequant_gemm(qweight: torch.Tensor, d_in: int, scales_f16: torch.Tensor,
                      zeros_f16: torch.Tensor, group_size: int, X: torch.Tensor, Y: torch.Tensor,
                      dev_status: torch.Tensor | None = None) -> None:
    """Y [m, d_out] (fp32) = X [m, d_in] (fp16) @ W_hat^T from the packed 4-bit layer."""
    for t, nm in ((qweight, "qweight"), (scales_f16, "scales_f16"), (zeros_f16, "zeros_f16"),
                  (X, "X"), (Y, "Y")):
        _dev(t, nm)
    if X.dtype != torch.float16 or Y.dtype != torch.float32:
        raise ValueError("X must be float16 and Y float32")
    X2 = X.reshape(-1, X.shape[-1])
    Y2 = Y.reshape(-1, Y.shape[-1])
    _row_major(X2, "X")
    _row_major(Y2, "Y")
    rc = _lib.gptq_dequant_gemm(_ptr(qweight), qweight.shape[0], int(d_in), _ptr(scales_f16),
                                _ptr(zeros_f16), scales_f16.shape[1], int(group_size), _ptr(X2),
                                X2.shape[0], X2.stride(0), _ptr(Y2), Y2.stride(0),
                                _ptr(dev_status), _stream())
    _check(rc, "gptq_dequant_gemm")


def rtn_quantize(W: torch.Tensor, params: gptq_params, codes: torch.Tensor, scales: torch.Tensor,
                 zeros: torch.Tensor) -> None:
    _dev(W, "W", None, 2)
    _row_major(W, "W")
    n, d = W.shape
    G = 1 if params.group_size == -1 else d // params.group_size
    if codes.shape != (n, d) or scales.shape != (n, G) or zeros.shape != (n, G):
        raise ValueError("output shapes disagree with W / group_size")
    rc = _lib.rtn_quantize(_ptr(W), _dtype_code(W), W.stride(0), n, d, ctypes.byref(params),
                           _ptr(codes), _ptr(scales), _ptr(zeros), _stream())
    _check(rc, "rtn_quantize")


def gptq_gemm_f32(A: torch.Tensor, B: torch.Tensor, C: torch.Tensor, alpha: float = 1.0,
                  beta: float = 0.0, trans_a: bool = False, trans_b: bool = False,
                  dev_status: torch.Tensor | None = None) -> None:
    """C = alpha op(A) op(B) + beta C (fp32, row-major tensors; op = transpose when trans_*)."""
    for t, name in ((A, "A"), (B, "B"), (C, "C")):
        _dev(t, name, torch.float32, 2)
        _row_major(t, name)
    M = A.shape[1] if trans_a else A.shape[0]
    K = A.shape[0] if trans_a else A.shape[1]
    Kb = B.shape[1] if trans_b else B.shape[0]
    N = B.shape[0] if trans_b else B.shape[1]
    if Kb != K or tuple(C.shape) != (M, N):
        raise ValueError("shapes of A, B and C do not form a product")
    rc = _lib.gptq_gemm_f32(M, N, K, float(alpha), _ptr(A), A.stride(0), int(bool(trans_a)),
                            _ptr(B), B.stride(0), int(bool(trans_b)), float(beta), _ptr(C),
                            C.stride(0), _ptr(dev_status), _stream())
    _check(rc, "gptq_gemm_f32")


def gptq_quantize_pack_layer(W: torch.Tensor, U: torch.Tensor, perm: torch.Tensor,
                             dead: torch.Tensor, params: gptq_params, qweight: torch.Tensor,
                             scales_f16: torch.Tensor, zeros_f16: torch.Tensor,
                             scales: torch.Tensor, zeros: torch.Tensor, g_idx: torch.Tensor,
                             ws: torch.Tensor, dev_status: torch.Tensor | None = None) -> None:
    """The column sweep writing the packed layer directly (qweight int32/uint32 words, fp16 bits
    of scales and zeros as int16 tensors), plus fp32 scales/zeros and g_idx."""
    _dev(W, "W", None, 2)
    _row_major(W, "W")
    n, d = W.shape
    _dev(U, "U", torch.float32, 2)
    _dev(scales, "scales", torch.float32, 2)
    _dev(zeros, "zeros", torch.float32, 2)
    _dev(g_idx, "g_idx", torch.int32, 1)
    _dev(ws, "ws")
    for t, name in ((qweight, "qweight"), (scales_f16, "scales_f16"), (zeros_f16, "zeros_f16")):
        _dev(t, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    G = 1 if params.group_size == -1 else d // params.group_size
    if qweight.element_size() != 4 or tuple(qweight.shape) != (n, d * params.bits // 32):
        raise ValueError("qweight must be 32-bit words [d_out, d_in * bits / 32]")
    for t in (scales, zeros, scales_f16, zeros_f16):
        if tuple(t.shape) != (n, G) or not t.is_contiguous():
            raise ValueError("scales / zeros (fp32 and fp16) must be contiguous [d_out, n_groups]")
    if scales_f16.element_size() != 2 or zeros_f16.element_size() != 2:
        raise ValueError("scales_f16 / zeros_f16 hold 16-bit patterns")
    if U.shape != (d, d) or g_idx.numel() != d:
        raise ValueError("U must be d_in x d_in and g_idx must have d_in entries")
    rc = _lib.gptq_quantize_pack_layer(_ptr(W), _dtype_code(W), W.stride(0), n, d, _ptr(U),
                                       _ptr(perm), _ptr(dead), ctypes.byref(params),
                                       _ptr(qweight), _ptr(scales_f16), _ptr(zeros_f16),
                                       _ptr(scales), _ptr(zeros), _ptr(g_idx), _ptr(ws),
                                       ws.numel() * ws.element_size(), _ptr(dev_status),
                                       _stream())
    _check(rc, "gptq_quantize_pack_layer")
