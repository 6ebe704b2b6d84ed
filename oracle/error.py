"""The layer-wise objective ||W X - W_hat X||_F^2 — oracle.

[INT4-GPTQ] §The Quantization Error and Layerwise Objective and [GPTQ-MATH] §The Layer-Wise
Reconstruction Problem: L(W_hat) = ||(W - W_hat) X||_F^2, a sum of independent row terms.
With delta = W - W_hat (one row) and H = 2 X X^T, ||delta X||^2 = delta (H/2) delta^T
([GPTQ-MATH] §Second-Order Taylor Expansion: E = 1/2 delta^T H delta), so the error of a whole
layer is 1/2 sum_rows delta_r H delta_r^T with the undamped H.

Pinned by: the H form against the direct product ||X_tm delta^T||_F^2 on small inputs.
"""
from __future__ import annotations

import numpy as np

from .hessian import as_f64


def dequant_matrix(codes: np.ndarray, S: np.ndarray, Z: np.ndarray, g_idx: np.ndarray) -> np.ndarray:
    """W_hat [n, d] in original column order: s[g_idx[c]] * (code[c] - z[g_idx[c]])."""
    g_idx = np.asarray(g_idx, np.int64)
    S = np.asarray(S, np.float64)
    Z = np.asarray(Z, np.float64)
    return S[:, g_idx] * (np.asarray(codes, np.float64) - Z[:, g_idx])


def layer_error(W: np.ndarray, W_hat: np.ndarray, H: np.ndarray) -> float:
    """1/2 sum_r delta_r H delta_r^T with the undamped H = 2 X X^T."""
    D = np.asarray(W, np.float64) - np.asarray(W_hat, np.float64)
    return float(0.5 * np.sum((D @ np.asarray(H, np.float64)) * D))


def row_errors(W: np.ndarray, W_hat: np.ndarray, H: np.ndarray) -> np.ndarray:
    D = np.asarray(W, np.float64) - np.asarray(W_hat, np.float64)
    return 0.5 * np.sum((D @ np.asarray(H, np.float64)) * D, axis=1)


def layer_error_direct(W: np.ndarray, W_hat: np.ndarray, X_tm: np.ndarray) -> float:
    """||(W - W_hat) X||_F^2 computed as ||X_tm (W - W_hat)^T||_F^2 (small inputs)."""
    D = np.asarray(W, np.float64) - np.asarray(W_hat, np.float64)
    return float(np.sum((np.asarray(X_tm, np.float64) @ D.T) ** 2))


def row_errors_direct(W_rows: np.ndarray, W_hat_rows: np.ndarray, X_tm: np.ndarray,
                      chunk: int = 16384) -> np.ndarray:
    """Per-row ||(w - w_hat) X||^2 for a few rows, streaming X_tm in token chunks."""
    D = (np.asarray(W_rows, np.float64) - np.asarray(W_hat_rows, np.float64)).T   # [d, r]
    out = np.zeros(D.shape[1])
    for t0 in range(0, X_tm.shape[0], chunk):
        y = as_f64(X_tm[t0:t0 + chunk]) @ D
        out += np.sum(y * y, axis=0)
    return out
