"""Layer Hessian H = 2 X X^T — oracle.

[INT4-GPTQ] §The Quantization Error and Layerwise Objective: H = 2 X X^T in R^{d_in x d_in}.
[Q-INT8] §Where the Hessian comes from: E = delta X X^T delta^T, second derivative 2 X X^T.
[GPTQ-MATH] §Second-Order Taylor Expansion and the Hessian: H = 2 X X^T, independent of W.

X is given token-major, X_tm [N, d_in] (the pages' X is X_tm^T), so H_ij = 2 sum_t X_ti X_tj.
Inputs are widened exactly to float64 before any arithmetic.

Pinned by: a hand-computed 3-token, 2-channel case (tests/golden/hessian_hand.txt), pure-Python
triple-loop brute force on tiny inputs, diag(H) = 2 sum_t X_t^2, symmetry, positive
semi-definiteness.
"""
from __future__ import annotations

import numpy as np


def as_f64(x) -> np.ndarray:
    """Exact float64 copy of a numpy array or of a CPU torch tensor (bf16 included)."""
    if hasattr(x, "double") and hasattr(x, "numpy"):
        return x.double().numpy()
    return np.asarray(x, np.float64)


def hessian(X_tm: np.ndarray, chunk: int = 16384) -> np.ndarray:
    """H = 2 X^T X over token-major X (float64), summed over token chunks.

    H is symmetric, so each chunk adds only its upper triangle, with the BLAS symmetric rank-k
    update (dsyrk) as the library step; the lower triangle is the mirror of the upper one."""
    from scipy.linalg import blas
    N, d = X_tm.shape
    H = np.zeros((d, d), np.float64, order="F")
    for t0 in range(0, N, chunk):
        xc = np.ascontiguousarray(as_f64(X_tm[t0:t0 + chunk]))
        # xc is [t, d] row-major, i.e. the column-major [d, t] matrix A = xc^T; C += A A^T.
        H = blas.dsyrk(1.0, xc.T, beta=1.0, c=H, trans=0, lower=0, overwrite_c=1)
    H = np.triu(H)
    H += np.triu(H, 1).T
    return 2.0 * H


def hessian_loops(X_tm) -> list[list[float]]:
    """Brute force: H_ij = 2 * sum_t X_ti X_tj with explicit Python loops (tiny inputs only)."""
    rows = [[float(v) for v in r] for r in np.asarray(X_tm, np.float64)]
    d = len(rows[0]) if rows else 0
    H = [[0.0] * d for _ in range(d)]
    for i in range(d):
        for j in range(d):
            acc = 0.0
            for r in rows:
                acc += r[i] * r[j]
            H[i][j] = 2.0 * acc
    return H


def hessian_rows(X_tm: np.ndarray, rows: np.ndarray, chunk: int = 16384) -> np.ndarray:
    """Selected rows H[rows, :] (float64), for sampled checks at sizes where full H is costly."""
    N, d = X_tm.shape
    rows = np.asarray(rows)
    out = np.zeros((rows.size, d), np.float64)
    for t0 in range(0, N, chunk):
        xc = as_f64(X_tm[t0:t0 + chunk])
        out += xc[:, rows].T @ xc
    return 2.0 * out


def hessian_diag(X_tm: np.ndarray, chunk: int = 16384) -> np.ndarray:
    """diag(H)_j = 2 sum_t X_tj^2 ([GPTQ-MATH] §Activation Ordering, step 1)."""
    N, d = X_tm.shape
    out = np.zeros(d, np.float64)
    for t0 in range(0, N, chunk):
        xc = as_f64(X_tm[t0:t0 + chunk])
        out += np.einsum("td,td->d", xc, xc)
    return 2.0 * out
