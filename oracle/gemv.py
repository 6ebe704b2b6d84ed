"""Dequantizing matrix-vector product on the packed format (the W4A16 / W3A16 consumer) — oracle.

[GPTQ-MATH] §Inference Execution and Modern Kernel Architectures: at inference the packed codes
are unpacked and dequantized, w_hat = (q - z) * s with the FP16 scale and zero, and multiplied
with FP16 activations, accumulating in higher precision (the fused dequantize-and-GEMV of
low-batch decoding). Here: Y[b, r] = sum_c (code[r, c] - z[r, g_idx[c]]) * s[r, g_idx[c]] * X[b, c]
in float64, with s and z the FP16 values stored by the pack format and X the FP16 activations
widened exactly.

Pinned by: a hand-computed 2 x 8 int4 case (tests/golden/gemv_hand.txt), agreement with the
dequantized matrix built directly from the codes (not through the packed words), and linearity
in X.
"""
from __future__ import annotations

import numpy as np

from . import pack as pk


def fp16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def dequant_gemv(qweight: np.ndarray, scales_f16: np.ndarray, zeros_f16: np.ndarray,
                 g_idx: np.ndarray, d: int, bits: int, X: np.ndarray) -> np.ndarray:
    """Y [B, n] = X [B, d] @ W_hat^T with W_hat unpacked from qweight [n, words] (float64)."""
    codes = pk.unpack_rows(np.asarray(qweight), d, bits).astype(np.float64)
    S = fp16_bits_to_f64(scales_f16)
    Z = fp16_bits_to_f64(zeros_f16)
    g_idx = np.asarray(g_idx, np.int64)
    W_hat = (codes - Z[:, g_idx]) * S[:, g_idx]
    X = np.atleast_2d(np.asarray(X, np.float64))
    return X @ W_hat.T
