"""Pins for oracle/hessian.py (no GPU)."""
import numpy as np

from conftest import parse_matrix, read_golden
from oracle import hessian as hs


def test_hand_case():
    g = read_golden("hessian_hand.txt")
    X = np.array(parse_matrix(g["X_tm"]))
    np.testing.assert_array_equal(hs.hessian(X), np.array(parse_matrix(g["H"])))
    assert hs.hessian_loops(X) == parse_matrix(g["H"])


def test_brute_force_loops():
    rng = np.random.default_rng(0)
    X = rng.normal(size=(37, 9)) * rng.lognormal(0, 0.5, 9)
    np.testing.assert_allclose(hs.hessian(X, chunk=8), np.array(hs.hessian_loops(X)),
                               rtol=1e-13, atol=1e-12)


def test_symmetric_psd_and_diag():
    """H is symmetric PSD; diag(H)_j = 2 sum_t X_tj^2 ([GPTQ-MATH] §Activation Ordering)."""
    rng = np.random.default_rng(1)
    X = np.abs(rng.normal(size=(500, 40)))
    H = hs.hessian(X, chunk=128)
    np.testing.assert_array_equal(H, H.T)
    assert np.linalg.eigvalsh(H).min() > -1e-9 * np.abs(H).max()
    np.testing.assert_allclose(np.diag(H), 2 * (X ** 2).sum(0), rtol=1e-14)
    np.testing.assert_allclose(hs.hessian_diag(X, chunk=64), np.diag(H), rtol=1e-14)
    rows = np.array([3, 0, 39])
    np.testing.assert_allclose(hs.hessian_rows(X, rows, chunk=77), H[rows], rtol=1e-13)


def test_rank_deficient_dead_channel():
    """A channel that never fires gives a zero row and column of H."""
    rng = np.random.default_rng(2)
    X = rng.normal(size=(64, 6))
    X[:, 4] = 0
    H = hs.hessian(X)
    assert np.all(H[4] == 0) and np.all(H[:, 4] == 0)
