"""Helpers for the GPU parity tests: run the CUDA path through the C ABI, compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from oracle import error as er
from oracle import hessian as hs


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a CPU/GPU bf16 or fp32 tensor."""
    return t.detach().to("cpu", torch.float64).numpy()


def make_inputs(n, d, N, seed, x_dtype=torch.bfloat16, w_dtype=torch.bfloat16, chan_sigma=1.0,
                outlier_frac=0.001, outlier_mult=20.0, half_normal=False, w_sigma=0.02):
    import layer_inputs as li
    X = li.activations(N, d, chan_sigma=chan_sigma, outlier_frac=outlier_frac,
                       outlier_mult=outlier_mult, half_normal=half_normal, dtype=x_dtype,
                       seed=seed)
    W = li.weight(n, d, w_sigma, w_dtype, seed=seed + 1)
    return W, X


def gpu_pipeline(W, X=None, H=None, bits=4, group_size=128, sym=False, act_order=False,
                 perm=None, percdamp=0.01, static_groups=False):
    """Hessian -> prepare -> sweep on the GPU. Returns host numpy arrays."""
    import post_weight_quantization_18_b200 as G
    Wd = W.cuda()
    Hd = None
    if H is not None:
        Hd = torch.as_tensor(H, dtype=torch.float32).cuda().contiguous()
    Xd = X.cuda() if X is not None else None
    pd = torch.as_tensor(perm, dtype=torch.int32).cuda() if perm is not None else None
    out = G.quantize_layer(Wd, X=Xd, H=Hd, bits=bits, group_size=group_size, sym=sym,
                           act_order=act_order, perm=pd, percdamp=percdamp,
                           static_groups=static_groups)
    torch.cuda.synchronize()
    return dict(codes=out.codes.cpu().numpy(), S=out.scales.cpu().numpy().astype(np.float64),
                Z=out.zeros.cpu().numpy().astype(np.float64),
                g_idx=out.g_idx.cpu().numpy().astype(np.int64),
                perm=out.perm.cpu().numpy().astype(np.int64), dead=out.dead.cpu().numpy())


def layer_err(W64, res, H64):
    return er.layer_error(W64, er.dequant_matrix(res["codes"], res["S"], res["Z"], res["g_idx"]),
                          H64)


def trajectory_check(W64, U64, perm, dead, codes, S, Z, bits, group_size, sym, tau=1e-3,
                     static_groups=False):
    """Teacher-forced validity of a sweep result (tests only).

    Runs the column sweep in float64 with the oracle's U, but follows the decisions under test:
    at every column the compensated weight w_j is computed exactly from the original W and the
    previous codes, and the code under test must be the quantizer's rounding of w_j (within
    `tau` of a half-step tie; clamped ends may lie anywhere beyond). Group statistics are
    recomputed from the current weights and compared with the scales/zeros under test. Several
    results are valid when a weight lies on a tie; this checks the one given without the
    cascade that a single tie decision causes in the later columns of its row.
    With static_groups the parameters are the ones given (original group of each column), and
    they are checked once against the statistics of the original, dead-fixed weights.
    Returns dict(bad_codes, max_excess, s_rel, z_bad).
    """
    from oracle import quantizer as qz
    n, d = W64.shape
    W = np.array(W64[:, perm], np.float64)
    W[:, np.asarray(dead, bool)] = 0.0
    C = np.asarray(codes)[:, perm].astype(np.float64)
    g = d if group_size == -1 else group_size
    maxq = 2 ** bits - 1
    bad = 0
    excess = 0.0
    s_rel = 0.0
    z_bad = 0
    if static_groups:
        W_orig = np.empty_like(W)
        W_orig[:, np.asarray(perm)] = W
        for gi in range(d // g):
            so, zo = qz.params_from_values(W_orig[:, gi * g:(gi + 1) * g], bits, sym)
            s_rel = max(s_rel, float(np.max(np.abs(so - S[:, gi]) / so)))
            if not sym:
                mn = np.min(W_orig[:, gi * g:(gi + 1) * g], axis=1)
                xz = -mn / S[:, gi]
                z_bad += int(np.sum((zo != Z[:, gi]) &
                                    (np.abs(np.abs(xz - np.floor(xz)) - 0.5) > tau)))
    for j in range(d):
        gi = 0 if group_size == -1 else j // g
        if static_groups:
            gi = int(perm[j]) // g
        s, z = S[:, gi], Z[:, gi]
        if not static_groups and ((group_size == -1 and j == 0) or
                                  (group_size != -1 and j % g == 0)):
            so, zo = qz.params_from_values(W[:, j:] if group_size == -1 else W[:, j:j + g],
                                           bits, sym)
            s_rel = max(s_rel, float(np.max(np.abs(so - s) / so)))
            if not sym:
                mn = np.min(W[:, j:] if group_size == -1 else W[:, j:j + g], axis=1)
                xz = -mn / s
                z_bad += int(np.sum((zo != z) & (np.abs(np.abs(xz - np.floor(xz)) - 0.5) > tau)))
        x = W[:, j] / s + z
        c = C[:, j]
        lo = np.where(c == 0, -np.inf, c - 0.5 - tau)
        hi = np.where(c == maxq, np.inf, c + 0.5 + tau)
        viol = (x < lo) | (x > hi)
        bad += int(viol.sum())
        if viol.any():
            excess = max(excess, float(np.max(np.maximum(lo - x, x - hi)[viol])))
        wh = s * (c - z)
        err = (W[:, j] - wh) / U64[j, j]
        W[:, j + 1:] -= np.outer(err, U64[j, j + 1:])
    return dict(bad_codes=bad, max_excess=excess, s_rel=s_rel, z_bad=z_bad)


def compare_with_oracle(W, X, bits=4, group_size=128, sym=False, act_order=False,
                        given_perm=False, code_agree=0.99, err_rtol=1e-3, static_groups=False):
    """Full GPU pipeline vs the oracle on the same seeded inputs.

    Asserts: every GPU code is a valid rounding along its own trajectory (trajectory_check,
    tie band 1e-3 step), scales within 1e-4 relative, layer error within err_rtol of the
    oracle's, plain code agreement >= code_agree (a tie decided differently in fp32 changes the
    later codes of that row, so plain agreement is a weaker, cascade-sensitive measure)."""
    W64, X64 = f64(W), f64(X)
    H64 = hs.hessian(X64)
    ora = oracle.gptq_layer(W64, H64, bits, group_size, sym, act_order=act_order,
                            static_groups=static_groups)
    perm = ora["perm"] if given_perm else None
    gpu = gpu_pipeline(W, X, bits=bits, group_size=group_size, sym=sym,
                       act_order=act_order and not given_perm, perm=perm,
                       static_groups=static_groups)
    if act_order and not given_perm:
        assert_valid_desc_order(gpu["perm"], np.diag(H64))
    agree = float(np.mean(gpu["codes"] == ora["codes"]))
    e_gpu, e_ora = layer_err(W64, gpu, H64), layer_err(W64, ora, H64)
    rel = abs(e_gpu - e_ora) / e_ora
    assert np.all(gpu["codes"] < 2 ** bits)
    from oracle import prepare as prep
    U64 = prep.prepare(H64, W64[:1], 0.01, perm=gpu["perm"])["U"]
    tc = trajectory_check(W64, U64, gpu["perm"], gpu["dead"], gpu["codes"], gpu["S"], gpu["Z"],
                          bits, group_size, sym, static_groups=static_groups)
    msg = f"agree {agree:.6f}, rel err {rel:.2e}, trajectory {tc}"
    assert tc["bad_codes"] == 0 and tc["z_bad"] == 0, msg
    assert tc["s_rel"] <= 1e-4, msg
    assert rel <= err_rtol, msg
    assert agree >= code_agree, msg
    return agree, rel, gpu, ora


def assert_valid_desc_order(perm, diag, rtol=1e-5):
    """perm must be a permutation sorting diag descending, up to near-ties (fp32 vs fp64 H)."""
    assert sorted(perm.tolist()) == list(range(len(diag)))
    v = diag[perm]
    bad = v[1:] > v[:-1] * (1 + rtol) + 1e-30
    assert not np.any(bad), f"{int(bad.sum())} out-of-order pairs"
