"""The GPTQ column sweep — oracle (float64).

Every route quantizes the columns of the (already permuted, dead-fixed) working matrix W in the
fixed order 0..d-1, the same order for every row ([GPTQ-MATH] §1 Arbitrary Order Quantization),
and after each column compensates the not-yet-quantized columns of every row with the OBS rule
  delta_F = -(w_q - quant(w_q)) / [H_F^-1]_qq * (H_F^-1)_{:,q}
([INT4-GPTQ] §The GPTQ Update Rule; [Q-INT8] §Where the Hessian comes from; [GPTQ-MATH]
§Lagrangian Derivation).

Group statistics (reading of the pages, whose pseudocode calls a group quantizer on a single
column): when the sweep reaches position k with k % g == 0, (s, z) of group [k, k+g) are taken
from the current, already compensated values of those g columns of each row ([INT4-GPTQ]
§Group Quantization gives the statistics of a run of g consecutive weights). With one scale per
row (group_size == -1) the statistics come from the whole row at the start of the sweep.

Static groups (the pre-computed group option listed among GPTQ's hyperparameters next to
act-order): the groups are runs of g columns in the original column order, their (s, z) are
taken once from the original (dead-column-fixed) weights before the sweep, and a column swept at
position j uses the parameters of its original group. The routes take them as `static`.

Precision: the compensation runs in float64; the integer decisions (the group's zero point and
every code) and the group scale are taken in float32, from the float64 compensated weights
rounded once to float32, with IEEE division and round-half-to-even: the pages' quantizer is
float32 tensor code, and a decision that floating point takes must be taken in the same
precision as the kernel under test takes it (the RTN and quantize-given-scales paths of
quantizer.py already run in float32).

Routes
  sweep_obs       OBS update with the explicit inverse Hessian H_F^-1, downdated after every
                  column by the rank-1 formula of [GPTQ-MATH] §Recursive Inverse Hessian
                  Updating. No Cholesky factor, no blocking.
  sweep_chol      the same sweep with rows of U (H^-1 = U^T U): err = (w_j - w_hat_j)/U_jj,
                  w_k -= err * U_jk for k > j ([GPTQ-MATH] §3 Cholesky Decomposition).
  sweep_blocked   sweep_chol with lazy batch updates: inside a block of B columns eager updates,
                  after the block W[:, i2:] -= Err_B U[i1:i2, i2:] ([GPTQ-MATH] §2 Lazy Batch
                  Updates, read with U in place of H^-1 — the only reading under which the lazy
                  form equals the eager one).
  sweep_lstsq     brute force that never forms H^-1: before quantizing column j, the free
                  weights are the least-squares optimum of the damped objective given the
                  already-quantized prefix. Tiny inputs only.

Pinned by: the four routes agreeing (codes identical, also with static groups); H = I reducing
to RTN (with static groups in any column order, the RTN of the original weights); the closed-form
saliency Delta E_q of [GPTQ-MATH] §Minimal Error Penalty for one quantized column; invariance of
the codes to scaling H by 4; GPTQ error <= RTN error on the small workload.
"""
from __future__ import annotations

import numpy as np

from . import quantizer as qz


def _decide_params(vals: np.ndarray, bits: int, sym: bool):
    """(s, z) of each row of vals, decided in float32 (see the module docstring)."""
    s, z = qz.params_from_values(np.asarray(vals, np.float64).astype(np.float32), bits, sym)
    return s.astype(np.float64), z.astype(np.float64)


def static_group_params(W_orig: np.ndarray, bits: int, group_size: int, sym: bool):
    """(S, Z) [n, G] of the runs of group_size columns of W in its original column order."""
    n, d = W_orig.shape
    G = (d + group_size - 1) // group_size
    S = np.zeros((n, G))
    Z = np.zeros((n, G))
    for gi in range(G):
        S[:, gi], Z[:, gi] = _decide_params(W_orig[:, gi * group_size:(gi + 1) * group_size],
                                            bits, sym)
    return S, Z


class _Groups:
    """Group bookkeeping shared by the routes (statistics over current values at group start,
    or fixed static parameters with a group per sweep column)."""

    def __init__(self, n: int, d: int, bits: int, group_size: int, sym: bool, W0: np.ndarray,
                 static=None):
        self.bits, self.sym = bits, sym
        self.g = d if group_size == -1 else group_size
        self.per_row = group_size == -1
        self.gid = None
        if static is not None:  # (S [n, G], Z [n, G], group of each sweep column [d])
            S, Z, gid = static
            self.S = np.array(S, np.float64, copy=True)
            self.Z = np.array(Z, np.float64, copy=True)
            self.gid = np.asarray(gid, np.int64)
            return
        G = 1 if self.per_row else (d + self.g - 1) // self.g
        self.S = np.zeros((n, G))
        self.Z = np.zeros((n, G))
        if self.per_row:
            s, z = _decide_params(W0, bits, sym)
            self.S[:, 0], self.Z[:, 0] = s, z

    def at(self, W: np.ndarray, j: int):
        """(s, z) for column j, computing the group's statistics when j starts a group."""
        if self.gid is not None:
            return self.S[:, self.gid[j]], self.Z[:, self.gid[j]]
        if self.per_row:
            return self.S[:, 0], self.Z[:, 0]
        gi = j // self.g
        if j % self.g == 0:
            s, z = _decide_params(W[:, j:j + self.g], self.bits, self.sym)
            self.S[:, gi], self.Z[:, gi] = s, z
        return self.S[:, gi], self.Z[:, gi]


def _quant_col(W, j, grp):
    """Code of column j decided in float32 from the float64 compensated weights; w_hat in
    float64 (exact: s is a float32 value and q - z a small integer)."""
    s, z = grp.at(W, j)
    q = qz.quantize(W[:, j].astype(np.float32), s.astype(np.float32), z.astype(np.float32),
                    grp.bits).astype(np.float64)
    return q, qz.dequantize(q, s, z)


def sweep_obs(W: np.ndarray, H_inv: np.ndarray, bits: int, group_size: int, sym: bool,
              n_steps: int | None = None, static=None):
    """OBS sweep with the explicit, recursively downdated inverse Hessian.

    n_steps stops after that many columns (the returned W then holds the quantized prefix and
    the compensated, still free remainder)."""
    W = np.array(W, np.float64, copy=True)
    Hi = np.array(H_inv, np.float64, copy=True)
    n, d = W.shape
    grp = _Groups(n, d, bits, group_size, sym, W, static)
    codes = np.zeros((n, d), np.uint8)
    for j in range(d if n_steps is None else n_steps):
        q, wh = _quant_col(W, j, grp)
        codes[:, j] = q.astype(np.uint8)
        # delta_F = -(w_j - w_hat_j) / [H_F^-1]_jj * (H_F^-1)_{F, j}, F = {j, ..., d-1}
        e = (W[:, j] - wh) / Hi[j, j]
        W[:, j:] -= np.outer(e, Hi[j:, j])
        # H_{F\j}^-1 = (H_F^-1)_{F\j,F\j} - (H_F^-1)_{F\j,j} (H_F^-1)_{j,F\j} / [H_F^-1]_jj
        Hi[j + 1:, j + 1:] -= np.outer(Hi[j + 1:, j], Hi[j, j + 1:]) / Hi[j, j]
    return codes, grp.S, grp.Z, W


def sweep_chol(W: np.ndarray, U: np.ndarray, bits: int, group_size: int, sym: bool,
               static=None):
    """Unblocked sweep with rows of the upper Cholesky factor U of H^-1."""
    W = np.array(W, np.float64, copy=True)
    n, d = W.shape
    grp = _Groups(n, d, bits, group_size, sym, W, static)
    codes = np.zeros((n, d), np.uint8)
    Err = np.zeros((n, d))
    for j in range(d):
        q, wh = _quant_col(W, j, grp)
        codes[:, j] = q.astype(np.uint8)
        Err[:, j] = (W[:, j] - wh) / U[j, j]
        W[:, j + 1:] -= np.outer(Err[:, j], U[j, j + 1:])
        W[:, j] = wh
    return codes, grp.S, grp.Z, Err


def sweep_blocked(W: np.ndarray, U: np.ndarray, bits: int, group_size: int, sym: bool,
                  block_size: int = 128, static=None):
    """Blocked sweep: eager updates inside each block, one lazy update of the columns after it."""
    W = np.array(W, np.float64, copy=True)
    n, d = W.shape
    grp = _Groups(n, d, bits, group_size, sym, W, static)
    codes = np.zeros((n, d), np.uint8)
    Err = np.zeros((n, d))
    for i1 in range(0, d, block_size):
        i2 = min(d, i1 + block_size)
        for j in range(i1, i2):
            q, wh = _quant_col(W, j, grp)
            codes[:, j] = q.astype(np.uint8)
            Err[:, j] = (W[:, j] - wh) / U[j, j]
            W[:, j + 1:i2] -= np.outer(Err[:, j], U[j, j + 1:i2])
            W[:, j] = wh
        if i2 < d:
            W[:, i2:] -= Err[:, i1:i2] @ U[i1:i2, i2:]
    return codes, grp.S, grp.Z, Err


def sweep_lstsq(W0: np.ndarray, A: np.ndarray, bits: int, group_size: int, sym: bool,
                static=None):
    """Brute force with no inverse Hessian: A is any matrix with A^T A = H_damped (for example
    [sqrt(2) X_tm ; sqrt(lambda) I]), so the damped objective of a row is ||A (w - w0)||^2.

    Before column j is quantized, the free weights F = {j, ..., d-1} of every row are set to the
    least-squares optimum given the quantized prefix: delta_F = argmin ||A_P delta_P + A_F delta_F||.
    Then column j is quantized from those values. Tiny inputs only (one lstsq per column).
    """
    W0 = np.array(W0, np.float64, copy=True)
    n, d = W0.shape
    grp = _Groups(n, d, bits, group_size, sym, W0, static)
    codes = np.zeros((n, d), np.uint8)
    Wq = np.zeros((n, d))                  # dequantized prefix
    W = W0.copy()
    for j in range(d):
        if j > 0:
            dP = (Wq[:, :j] - W0[:, :j]).T                     # [j, n]
            rhs = -(A[:, :j] @ dP)                             # [m, n]
            dF, *_ = np.linalg.lstsq(A[:, j:], rhs, rcond=None)
            W[:, j:] = W0[:, j:] + dF.T
        q, wh = _quant_col(W, j, grp)
        codes[:, j] = q.astype(np.uint8)
        Wq[:, j] = wh
    return codes, grp.S, grp.Z
