"""Numerical preparation of the Hessian — oracle.

Steps, in the order of the layer walkthrough of [GPTQ-MATH] §GPTQ Algorithm Execution
Walkthrough (and §Activation Ordering for the optional permutation, which comes first):

  1. act-order (optional): pi = argsort(diag(H), descending); W <- W[:, pi], H <- H[pi][:, pi]
     ([GPTQ-MATH] §Activation Ordering (Act-Order / Desc-Act), workflow steps 1-3).
  2. dead columns: where diag(H) == 0 set H_jj = 1 and W[:, j] = 0 (walkthrough, step 1).
  3. damping: lambda = percdamp * mean(diag(H)), H <- H + lambda I
     ([GPTQ-MATH] §Hessian Damping and Numerical Regularization; walkthrough step 1).
  4. U = upper Cholesky factor of H^-1 by the walkthrough's three steps:
     L = chol(H), H^-1 = cholesky_inverse(L) = L^-T L^-1, U = chol(H^-1, upper) so H^-1 = U^T U
     ([GPTQ-MATH] §Cholesky Decomposition and Pre-computation; walkthrough step 2).

Readings: the act-order sort key is the raw diag(H) (before the dead-column fix and damping);
the sort is stable (equal keys keep the lower index first). The damping mean is taken after the
dead-column fix, as the walkthrough orders it.

Pinned by: U^T U H_damped = I; H = I gives U = I / sqrt(1 + percdamp) exactly; the Cholesky
identities of [GPTQ-MATH] §3 ([H_F^-1]_kj / [H_F^-1]_jj = U_jk / U_jj and [H_F^-1]_jj = U_jj^2,
with H_F^-1 from a direct inverse of each trailing block); lambda_min(H_damped) >= lambda; hand
cases for dead columns and for the stable descending order.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg


def act_order_perm(diag_h: np.ndarray) -> np.ndarray:
    """pi = argsort(diag(H)) descending, stable (ties keep the lower index first)."""
    return np.argsort(-np.asarray(diag_h, np.float64), kind="stable").astype(np.int64)


def dead_fix(H: np.ndarray, W: np.ndarray):
    """Dead input channels (diag(H) == 0): H_jj = 1 and W[:, j] = 0. Returns copies and the mask."""
    H = np.array(H, np.float64, copy=True)
    W = np.array(W, np.float64, copy=True)
    dead = np.diag(H) == 0
    idx = np.flatnonzero(dead)
    H[idx, idx] = 1.0
    W[:, dead] = 0.0
    return H, W, dead


def damp(H: np.ndarray, percdamp: float):
    """H + lambda I with lambda = percdamp * mean(diag(H)). Returns (H_damped, lambda)."""
    lam = percdamp * float(np.mean(np.diag(H)))
    Hd = np.array(H, np.float64, copy=True)
    idx = np.arange(Hd.shape[0])
    Hd[idx, idx] += lam
    return Hd, lam


def chol_lower(A: np.ndarray) -> np.ndarray:
    """Lower Cholesky factor L of a symmetric positive definite A (A = L L^T), by LAPACK's
    dpotrf. A is symmetric, so its row-major array read column-major is A itself."""
    from scipy.linalg import lapack
    c, info = lapack.dpotrf(np.asarray(A, np.float64).T, lower=1, clean=1, overwrite_a=0)
    if info != 0:
        raise np.linalg.LinAlgError(f"dpotrf: leading minor {info} is not positive definite")
    return np.ascontiguousarray(c)


def cholesky_inverse(L: np.ndarray) -> np.ndarray:
    """(L L^T)^-1 = L^-T L^-1 from the lower Cholesky factor L, by LAPACK's dpotri (the
    'cholesky_inverse' step of the walkthrough); the full symmetric matrix is returned."""
    from scipy.linalg import lapack
    inv, info = lapack.dpotri(np.asfortranarray(L), lower=1, overwrite_c=0)
    if info != 0:
        raise np.linalg.LinAlgError(f"dpotri: info {info}")
    inv = np.tril(inv)
    inv += np.tril(inv, -1).T
    return np.ascontiguousarray(inv)


def upper_chol_of_inverse(H_damped: np.ndarray):
    """The walkthrough's three steps. Returns (H_inv, U) with H_inv = U^T U, U upper."""
    L = chol_lower(H_damped)
    H_inv = cholesky_inverse(L)
    del L
    U = np.ascontiguousarray(chol_lower(H_inv).T)
    return H_inv, U


def prepare(H: np.ndarray, W: np.ndarray, percdamp: float = 0.01, act_order: bool = False,
            perm: np.ndarray | None = None):
    """Steps 1-4 above. `perm`, when given, replaces the act-order sort (a caller-chosen order).

    Returns dict(W=working W (float64, permuted, dead columns zeroed), H_damped, H_inv, U,
    perm, dead (in sweep order), lam).
    """
    H = np.asarray(H, np.float64)
    W = np.asarray(W, np.float64)
    d = H.shape[0]
    if perm is None:
        perm = act_order_perm(np.diag(H)) if act_order else np.arange(d, dtype=np.int64)
    perm = np.asarray(perm, np.int64)
    identity = np.array_equal(perm, np.arange(d))
    Hp = H if identity else H[np.ix_(perm, perm)]
    Wp = W if identity else W[:, perm]
    Hp, Wp, dead = dead_fix(Hp, Wp)
    Hd, lam = damp(Hp, percdamp)
    H_inv, U = upper_chol_of_inverse(Hd)
    return dict(W=Wp, H_damped=Hd, H_inv=H_inv, U=U, perm=perm, dead=dead, lam=lam)
