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
                 perm=None, percdamp=0.01, static_groups=False, U=None, dead=None):
    """Hessian -> prepare -> sweep on the GPU (or, given U, perm and dead, the sweep alone).
    Returns host numpy arrays."""
    import post_weight_quantization_18_b200 as G
    Wd = W.cuda()
    pd = torch.as_tensor(perm, dtype=torch.int32).cuda() if perm is not None else None
    if U is not None:
        n, d = W.shape
        Ud = torch.as_tensor(np.asarray(U), dtype=torch.float32).cuda().contiguous()
        dd = torch.as_tensor(np.asarray(dead), dtype=torch.uint8).cuda()
        p = G.make_params(bits, group_size, sym, G.GPTQ_ORDER_GIVEN, 128, percdamp,
                          static_groups)
        Gn = 1 if group_size == -1 else d // group_size
        codes = torch.empty((n, d), dtype=torch.uint8, device="cuda")
        S = torch.empty((n, Gn), dtype=torch.float32, device="cuda")
        Z = torch.empty((n, Gn), dtype=torch.float32, device="cuda")
        gi = torch.empty(d, dtype=torch.int32, device="cuda")
        ws = torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device="cuda")
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        G.gptq_quantize_layer(Wd, Ud, pd, dd, p, codes, S, Z, gi, ws, st)
        G.check_status(st)
        out = G.QuantizedLayer(codes, S, Z, gi, pd, dd, bits, group_size)
    else:
        Hd = None
        if H is not None:
            Hd = torch.as_tensor(H, dtype=torch.float32).cuda().contiguous()
        Xd = X.cuda() if X is not None else None
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


def first_divergence_ties(gpu, ora, bits, group_size, sym):
    """Explain the code differences of a GPU run against the oracle's, row by row.

    In GPTQ a decision taken differently (a rounding or a zero point near a tie) changes the
    compensation of every later column of its row, so the rest of the row may follow another,
    equally valid trajectory. For every row whose GPU codes differ from the oracle's this finds
    the first difference in sweep order and measures, on the oracle's trajectory, how far the
    decision there was from its rounding boundary, in quantization steps:
      * a code: x = w / s with w the oracle's compensated weight (w_hat + Err * U_jj); distance
        of x to the nearest half-integer;
      * a zero point that differs at the first differing group: the distance of -min / s, with
        the group's weights as they were when its statistics were taken.
    Both sides must be run in the same column order (gpu['perm'] == ora['perm']).
    Returns a list of (row, first sweep position, distance); empty when all codes agree."""
    perm = np.asarray(ora["perm"])
    assert np.array_equal(np.asarray(gpu["perm"]), perm)
    cg = np.asarray(gpu["codes"])[:, perm].astype(np.int64)
    co = np.asarray(ora["codes"])[:, perm].astype(np.int64)
    U, Err = ora["U"], ora["Err"]
    n, d = co.shape
    g = d if group_size == -1 else group_size
    out = []
    for r in np.flatnonzero(np.any(cg != co, axis=1)):
        j = int(np.argmax(cg[r] != co[r]))
        gi = 0 if group_size == -1 else j // g
        s, z = ora["S"][r, gi], ora["Z"][r, gi]
        if gpu["Z"][r, gi] != z and not sym:
            # zero point decided differently: -min / s over the group's weights as they were at
            # the group's start, w_k + sum_{j0 <= i < k} Err_i U_ik with w_k the value column k
            # was quantized from (w_hat_k + Err_k U_kk)
            j0 = gi * g
            Ug = U[j0:j0 + g, j0:j0 + g]
            eg = Err[r, j0:j0 + g]
            w = s * (co[r, j0:j0 + g] - z) + eg * np.diag(Ug) + eg @ np.triu(Ug, 1)
            x = -np.min(w) / s
        else:
            w = s * (co[r, j] - z) + Err[r, j] * U[j, j]
            x = w / s
        dist = abs((x - np.floor(x)) - 0.5)
        out.append((int(r), j, float(dist)))
    return out


def compare_with_oracle(W, X, bits=4, group_size=128, sym=False, act_order=False,
                        given_perm=False, code_agree=0.999, err_rtol=1e-3, static_groups=False,
                        tie_band=1e-4):
    """Full GPU pipeline vs the oracle on the same seeded inputs, with the layer acceptance:
      * layer error ||(W - W_hat) X||^2 (float64, undamped H) within err_rtol (1e-3) relative of
        the oracle's;
      * the sweep's decisions: the GPU sweep run on the oracle's U (rounded to fp32), order and
        dead columns gives the oracle's codes on >= code_agree (99.9 %) of the entries;
      * the full pipeline: codes equal on >= code_agree of the entries, or else every row that
        differs starts differing at a decision within tie_band of a step from its rounding
        boundary on the oracle's trajectory (first_divergence_ties): a tie decided the other
        way, after which the row follows its own valid trajectory;
      * every GPU code is a valid rounding along its own trajectory (trajectory_check, tie band
        1e-3 step), scales within 1e-4 relative.

    Act-order computed on the GPU (act_order and not given_perm): the GPU's permutation must
    sort the float64 diag(H) descending up to fp32 near-ties (assert_valid_desc_order) and its
    run must be a valid trajectory; the comparisons above then use a second GPU run given the
    oracle's permutation (GPTQ_ORDER_GIVEN), so that they measure the sweep and not the order of
    near-equal diagonal entries. Returns (agreement, relative error difference, gpu, oracle)."""
    from oracle import prepare as prep
    W64, X64 = f64(W), f64(X)
    H64 = hs.hessian(X64)
    ora = oracle.gptq_layer(W64, H64, bits, group_size, sym, act_order=act_order,
                            static_groups=static_groups)
    e_ora = layer_err(W64, ora, H64)

    def valid(gpu, tag):
        assert np.all(gpu["codes"] < 2 ** bits)
        U64 = prep.prepare(H64, W64[:1], 0.01, perm=gpu["perm"])["U"]
        tc = trajectory_check(W64, U64, gpu["perm"], gpu["dead"], gpu["codes"], gpu["S"],
                              gpu["Z"], bits, group_size, sym, static_groups=static_groups)
        assert tc["bad_codes"] == 0 and tc["z_bad"] == 0, (tag, tc)
        assert tc["s_rel"] <= 1e-4, (tag, tc)

    if act_order and not given_perm:
        own = gpu_pipeline(W, X, bits=bits, group_size=group_size, sym=sym, act_order=True,
                           static_groups=static_groups)
        assert_valid_desc_order(own["perm"], np.diag(H64))
        valid(own, "GPU act-order")
    perm = ora["perm"] if act_order else None
    gpu = gpu_pipeline(W, X, bits=bits, group_size=group_size, sym=sym, perm=perm,
                       static_groups=static_groups)
    valid(gpu, "pipeline")
    agree = float(np.mean(gpu["codes"] == ora["codes"]))
    rel = abs(layer_err(W64, gpu, H64) - e_ora) / e_ora
    msg = f"agree {agree:.6f}, rel err {rel:.2e}"
    assert rel <= err_rtol, msg
    if agree < code_agree:
        ties = first_divergence_ties(gpu, ora, bits, group_size, sym)
        assert ties and max(t[2] for t in ties) <= tie_band, (msg, ties)
    # the sweep on the oracle's own U, order and dead columns
    swp = gpu_pipeline(W, U=ora["U"], perm=ora["perm"], dead=ora["dead"], bits=bits,
                       group_size=group_size, sym=sym, static_groups=static_groups)
    agree_sweep = float(np.mean(swp["codes"] == ora["codes"]))
    assert agree_sweep >= code_agree, f"sweep on the oracle's U: agree {agree_sweep:.6f}"
    return agree, rel, gpu, ora


def assert_valid_desc_order(perm, diag, rtol=1e-5):
    """perm must be a permutation sorting diag descending, up to near-ties (fp32 vs fp64 H)."""
    assert sorted(perm.tolist()) == list(range(len(diag)))
    v = diag[perm]
    bad = v[1:] > v[:-1] * (1 + rtol) + 1e-30
    assert not np.any(bad), f"{int(bad.sum())} out-of-order pairs"
