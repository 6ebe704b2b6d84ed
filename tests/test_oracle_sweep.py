"""Pins for oracle/sweep.py and oracle/layer.py (no GPU)."""
import numpy as np
import pytest
import torch

import layer_inputs as li
import oracle
from oracle import error as er
from oracle import hessian as hs
from oracle import prepare as prep
from oracle import quantizer as qz
from oracle import sweep as sw


def _case(n=6, d=40, N=600, seed=0, half=False, dead=()):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(N, d))
    if half:
        X = np.abs(X)
    X *= rng.lognormal(0, 0.8, d)
    X[:, list(dead)] = 0
    W = rng.normal(0, 0.02, (n, d))
    return W, X, hs.hessian(X)


@pytest.mark.parametrize("bits,gs,sym,half", [(4, 8, False, False), (3, 16, False, True),
                                             (4, -1, True, True), (2, 8, True, False)])
def test_routes_agree(bits, gs, sym, half):
    """OBS-with-downdate == Cholesky rows == blocked (B in 1, 8, 16, d) == least squares."""
    W, X, H = _case(half=half, dead=(5,))
    P = prep.prepare(H, W, 0.01)
    ref = sw.sweep_obs(P["W"], P["H_inv"], bits, gs, sym)
    c, S, Z, Err = sw.sweep_chol(P["W"], P["U"], bits, gs, sym)
    np.testing.assert_array_equal(c, ref[0])
    np.testing.assert_allclose(S, ref[1], rtol=1e-9)
    for B in (1, 8, 16, 40):
        cb, Sb, Zb, Eb = sw.sweep_blocked(P["W"], P["U"], bits, gs, sym, B)
        np.testing.assert_array_equal(cb, c)
        np.testing.assert_allclose(Eb, Err, rtol=1e-9, atol=1e-12)
    # least squares on A with A^T A = H_damped (dead channel gets sqrt(1 + lambda))
    lam = P["lam"]
    diag_extra = np.sqrt(lam + P["dead"].astype(float))
    A = np.vstack([np.sqrt(2.0) * X[:, P["perm"]], np.diag(diag_extra)])
    np.testing.assert_allclose(A.T @ A, P["H_damped"], rtol=1e-12, atol=1e-9)
    cl, Sl, Zl = sw.sweep_lstsq(P["W"], A, bits, gs, sym)
    np.testing.assert_array_equal(cl, c)
    np.testing.assert_allclose(Sl, S, rtol=1e-8)


def test_identity_hessian_reduces_to_rtn():
    """H = I: U is diagonal, no compensation happens, GPTQ codes are RTN codes."""
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, (16, 256)).astype(np.float32)   # weights are fp32 or bf16 values
    for bits, gs, sym in [(4, 128, False), (3, 64, False), (4, -1, True)]:
        L = oracle.gptq_layer(W.astype(np.float64), np.eye(256), bits, gs, sym)
        R = oracle.rtn_layer(W, bits, gs, sym)
        np.testing.assert_array_equal(L["codes"], R["codes"])
        np.testing.assert_array_equal(L["S"], R["S"])
        np.testing.assert_array_equal(L["Z"], R["Z"])


def test_single_column_saliency():
    """[GPTQ-MATH] §Minimal Error Penalty: quantizing w_q and optimally compensating the rest
    raises 1/2 delta^T H delta by (w_q - quant(w_q))^2 / (2 [H^-1]_qq). With H = 2 X X^T the
    left side is ||delta X||^2, measured here directly from X. No damping, full-rank X."""
    W, X, H = _case(n=5, d=12, N=300, seed=2)
    H_inv = np.linalg.inv(H)
    c, S, Z, W1 = sw.sweep_obs(W, H_inv, 4, 12, False, n_steps=1)
    delta = W1 - W
    wq = qz.dequantize(c[:, 0].astype(np.float64), S[:, 0], Z[:, 0])   # the step's own w_hat
    assert np.all(np.abs(W[:, 0] - wq) <= S[:, 0] / 2 * (1 + 1e-6))   # a rounding of w_q
    expected = (W[:, 0] - wq) ** 2 / (2 * H_inv[0, 0])
    measured = np.sum((X @ delta.T) ** 2, axis=0)
    np.testing.assert_allclose(measured, expected, rtol=1e-9)


def test_obs_step_solves_constrained_qp():
    """[GPTQ-MATH] §Lagrangian Derivation: delta minimises 1/2 delta^T H delta subject to
    e_q^T delta = quant(w_q) - w_q; checked against a direct KKT solve."""
    W, X, H = _case(n=3, d=10, N=200, seed=3)
    Hd, _ = prep.damp(H, 0.01)
    c, S, Z, W1 = sw.sweep_obs(W, np.linalg.inv(Hd), 4, 10, False, n_steps=1)
    for r in range(3):
        target = W1[r, 0] - W[r, 0]
        K = np.zeros((11, 11))
        K[:10, :10] = Hd
        K[:10, 10] = K[10, :10] = np.eye(10)[0]
        sol = np.linalg.solve(K, np.r_[np.zeros(10), target])
        np.testing.assert_allclose(W1[r] - W[r], sol[:10], rtol=1e-8, atol=1e-14)


def test_scale_invariance():
    """Scaling H by 4 (exact in binary) leaves codes and scales bit-identical: the damping is
    relative and the OBS ratios are homogeneous of degree zero in H."""
    W, X, H = _case(n=8, d=64, seed=4, half=True)
    a = oracle.gptq_layer(W, H, 4, 16)
    b = oracle.gptq_layer(W, 4.0 * H, 4, 16)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["S"], b["S"])


def test_act_order_layer_unpermutes():
    """Act-order: codes come back in original column order and g_idx[pi[k]] = k // g."""
    W, X, H = _case(n=4, d=32, seed=5)
    L = oracle.gptq_layer(W, H, 4, 8, act_order=True)
    pi = L["perm"]
    assert sorted(pi.tolist()) == list(range(32))
    assert np.all(L["g_idx"][pi] == np.arange(32) // 8)
    P = prep.prepare(H, W, 0.01, act_order=True)
    c = sw.sweep_blocked(P["W"], P["U"], 4, 8, False, 128)[0]
    np.testing.assert_array_equal(L["codes"][:, pi], c)


def test_error_forms_agree():
    """1/2 sum delta H delta^T == ||(W - W_hat) X||_F^2 computed directly."""
    W, X, H = _case(n=7, d=24, seed=6)
    L = oracle.gptq_layer(W, H, 4, 8)
    Wh = er.dequant_matrix(L["codes"], L["S"], L["Z"], L["g_idx"])
    np.testing.assert_allclose(er.layer_error(W, Wh, H), er.layer_error_direct(W, Wh, X), rtol=1e-10)
    np.testing.assert_allclose(er.row_errors(W, Wh, H), er.row_errors_direct(W, Wh, X, chunk=64),
                               rtol=1e-10)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gptq_beats_rtn_on_small_workload(seed):
    """Expected (not a theorem): GPTQ's layer error is below RTN's on the small fp32 workload."""
    wl = li.WORKLOADS["tiny_256"]
    a = wl.acts[0]
    X = li.activations(a.n_tokens, a.d, chan_sigma=a.chan_sigma, dtype=torch.float32,
                       seed=a.seed + 100 * seed).numpy()
    W = li.weight(256, 256, 0.02, torch.float32, seed=wl.linears[0].seed + 100 * seed).numpy()
    H = hs.hessian(X)
    L = oracle.gptq_layer(W, H, 4, 128)
    R = oracle.rtn_layer(W, 4, 128)
    eg = er.layer_error(W, er.dequant_matrix(L["codes"], L["S"], L["Z"], L["g_idx"]), H)
    erx = er.layer_error(W, er.dequant_matrix(R["codes"], R["S"], R["Z"], R["g_idx"]), H)
    assert eg < erx


# ---- static groups: parameters from the original weights, groups in original column order ----

@pytest.mark.parametrize("bits,gs,sym", [(4, 8, False), (3, 16, True)])
def test_static_groups_routes_agree(bits, gs, sym):
    """With static groups the four routes still give identical codes (act-order permutation)."""
    W, X, H = _case(half=True, dead=(7,), seed=11)
    P = prep.prepare(H, W, 0.01, act_order=True)
    perm = P["perm"]
    assert not np.array_equal(perm, np.arange(len(perm)))
    W_orig = np.empty_like(P["W"])
    W_orig[:, perm] = P["W"]
    S0, Z0 = sw.static_group_params(W_orig, bits, gs, sym)
    static = (S0, Z0, perm // gs)
    ref = sw.sweep_obs(P["W"], P["H_inv"], bits, gs, sym, static=static)
    c, S, Z, Err = sw.sweep_chol(P["W"], P["U"], bits, gs, sym, static=static)
    np.testing.assert_array_equal(c, ref[0])
    for B in (1, 8, 40):
        np.testing.assert_array_equal(
            sw.sweep_blocked(P["W"], P["U"], bits, gs, sym, B, static=static)[0], c)
    lam = P["lam"]
    A = np.vstack([np.sqrt(2.0) * X[:, perm], np.diag(np.sqrt(lam + P["dead"].astype(float)))])
    np.testing.assert_array_equal(sw.sweep_lstsq(P["W"], A, bits, gs, sym, static=static)[0], c)
    # the parameters are fixed before the sweep: those of the original (dead-fixed) weights
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_array_equal(Z, Z0)


def test_static_groups_identity_hessian_is_rtn_in_any_order():
    """H = I with static groups: no compensation and the groups' parameters are RTN's, so the
    codes equal RTN of the original weights whatever the column order."""
    rng = np.random.default_rng(4)
    W = rng.normal(0, 0.02, (12, 96)).astype(np.float32)
    R = qz.rtn(W, 4, 32, False)
    for seed in range(3):
        perm = np.random.default_rng(seed).permutation(96)
        L = oracle.gptq_layer(W.astype(np.float64), np.eye(96), 4, 32, False, perm=perm,
                              static_groups=True)
        np.testing.assert_array_equal(L["codes"], R[0])
        np.testing.assert_array_equal(L["S"], R[1])
        np.testing.assert_array_equal(L["g_idx"], np.arange(96) // 32)


def test_static_groups_differ_from_dynamic_and_keep_error_low():
    """Static and dynamic groups are different methods (different codes); both compensate, so
    both stay below RTN's error on a correlated layer."""
    W, X, H = _case(n=16, d=64, N=800, seed=9)
    Ls = oracle.gptq_layer(W, H, 4, 16, act_order=True, static_groups=True)
    Ld = oracle.gptq_layer(W, H, 4, 16, act_order=True)
    assert not np.array_equal(Ls["codes"], Ld["codes"])
    R = oracle.rtn_layer(W, 4, 16)
    def err(L):
        return er.layer_error(W, er.dequant_matrix(L["codes"], L["S"], L["Z"], L["g_idx"]), H)
    assert err(Ls) < err(R) and err(Ld) < err(R)
