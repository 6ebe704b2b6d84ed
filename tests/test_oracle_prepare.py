"""Pins for oracle/prepare.py (no GPU)."""
import numpy as np

from oracle import hessian as hs
from oracle import prepare as prep


def _H(d=24, N=400, seed=0, half=False):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(N, d))
    if half:
        X = np.abs(X)
    X *= rng.lognormal(0, 1.0, d)
    return hs.hessian(X), X


def test_inverse_identity():
    """H^-1 = U^T U with U upper: U^T U H_damped = I."""
    H, _ = _H()
    Hd, lam = prep.damp(H, 0.01)
    H_inv, U = prep.upper_chol_of_inverse(Hd)
    assert np.allclose(U, np.triu(U))
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ Hd, np.eye(len(H)), atol=1e-10)


def test_identity_hessian():
    """H = I: lambda = 0.01, H_damped = 1.01 I, U = I / sqrt(1.01)."""
    H_inv, U = prep.upper_chol_of_inverse(prep.damp(np.eye(16), 0.01)[0])
    np.testing.assert_allclose(U, np.eye(16) / np.sqrt(1.01), rtol=1e-15, atol=0)


def test_cholesky_identities():
    """[GPTQ-MATH] §3: for F = {j..d-1}, [H_F^-1]_kj / [H_F^-1]_jj = U_jk / U_jj and
    [H_F^-1]_jj = U_jj^2, with H_F^-1 from a direct inverse of each trailing block of H."""
    H, _ = _H(d=20, half=True, seed=3)
    Hd, _ = prep.damp(H, 0.01)
    _, U = prep.upper_chol_of_inverse(Hd)
    for j in range(20):
        HFi = np.linalg.inv(Hd[j:, j:])
        np.testing.assert_allclose(HFi[0, 0], U[j, j] ** 2, rtol=1e-9)
        np.testing.assert_allclose(HFi[:, 0] / HFi[0, 0], U[j, j:] / U[j, j], rtol=1e-8, atol=1e-12)


def test_damping_bound():
    """[GPTQ-MATH] §Hessian Damping: lambda = percdamp * mean(diag H), lambda_min(H_damped) >= lambda."""
    rng = np.random.default_rng(4)
    X = rng.normal(size=(10, 30))           # rank 10 < d: H singular before damping
    H = hs.hessian(X)
    Hd, lam = prep.damp(H, 0.01)
    assert lam == 0.01 * np.mean(np.diag(H))
    assert np.linalg.eigvalsh(Hd).min() >= lam * (1 - 1e-9)


def test_dead_columns():
    """[GPTQ-MATH] walkthrough: diag(H) == 0 -> H_jj = 1 and W[:, j] = 0."""
    rng = np.random.default_rng(5)
    X = rng.normal(size=(50, 5))
    X[:, 2] = 0
    H = hs.hessian(X)
    W = rng.normal(size=(3, 5))
    H2, W2, dead = prep.dead_fix(H, W)
    assert dead.tolist() == [False, False, True, False, False]
    assert H2[2, 2] == 1.0 and np.all(W2[:, 2] == 0)
    np.testing.assert_array_equal(np.delete(W2, 2, 1), np.delete(W, 2, 1))
    assert np.all(H2[2, [0, 1, 3, 4]] == 0)


def test_act_order_stable_descending():
    """[GPTQ-MATH] §Activation Ordering: pi = argsort(diag(H), descending); ties keep index order."""
    assert prep.act_order_perm(np.array([3.0, 5.0, 3.0, 0.0, 5.0, 1.0])).tolist() == [1, 4, 0, 2, 5, 3]


def test_prepare_permutes_consistently():
    """prepare with act-order equals prepare of the explicitly permuted H and W."""
    H, _ = _H(d=12, seed=6)
    W = np.random.default_rng(6).normal(size=(4, 12))
    P = prep.prepare(H, W, 0.01, act_order=True)
    pi = P["perm"]
    assert np.all(np.diff(np.diag(H)[pi]) <= 0)
    Q = prep.prepare(H[np.ix_(pi, pi)], W[:, pi], 0.01, act_order=False)
    np.testing.assert_allclose(P["U"], Q["U"], rtol=1e-12)
    np.testing.assert_array_equal(P["W"], Q["W"])
