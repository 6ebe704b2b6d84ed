"""GPU parity at the full sizes of the five benchmark workloads, through the same C ABI calls
bench.py times (gptq_hessian_accumulate -> gptq_prepare_hinv -> gptq_quantize_layer -> gptq_pack).

For every Hessian of every workload the float64 oracle runs in full on the host: H = 2 X^T X
from all calibration tokens, the pages' three-step prepare (chol, cholesky_inverse, chol upper)
and the blocked sweep of a sample of rows of each linear that shares the Hessian (rows are
independent given H, so the sampled rows of several linears are swept together). Against it:
  * acceptance on the sampled rows: layer error ||(W - W_hat) X||^2 (float64, undamped H)
    within 1e-3 relative of the oracle's; codes equal on >= 99.9 % of the entries, or else every
    row that differs starts differing at a decision within TIE_BAND of a step from its rounding
    boundary on the oracle's trajectory (a tie decided the other way, after which the row
    follows its own valid trajectory: first_divergence_ties);
  * the sweep's decisions: the GPU sweep of the sampled rows run on the oracle's U (rounded to
    fp32), order and dead columns gives the oracle's codes on >= 99.9 % of the entries;
  * H: sampled rows against the oracle's H (relative Frobenius error <= 1e-4);
  * act-order: the GPU permutation sorts the float64 diag(H) descending up to fp32 near-ties;
    codes are then compared on a GPU run given the oracle's permutation (GPTQ_ORDER_GIVEN);
  * U: H_d (U^T U e_k) = e_k for sampled k (componentwise backward error <= 1e-4), and the
    trailing 1024 x 1024 block of U against the oracle's factor of that block;
  * sweep: the teacher-forced trajectory check on the sampled rows along the GPU's own U;
  * pack: bit-exact against the oracle's packing of the GPU codes; g_idx exact.
"""
import numpy as np
import pytest
import torch

import layer_inputs as li
import oracle
from gpu_util import assert_valid_desc_order, first_divergence_ties, trajectory_check
from oracle import error as er
from oracle import hessian as hs
from oracle import pack as pk
from oracle import prepare as prep

pytestmark = pytest.mark.gpu

CHUNK = 8192
# A row whose codes differ from the oracle's must start differing at a decision this close (in
# quantization steps) to its rounding boundary on the oracle's trajectory.
TIE_BAND = 1e-3


def _gpu_prepare(Xd, q, order):
    import post_weight_quantization_18_b200 as G
    d = Xd.shape[1]
    p = G.make_params(q.bits, q.group_size, q.sym, order, q.block_size, q.percdamp)
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    H = torch.empty((d, d), dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(H, Xd, 2.0, False, st)
    H_copy = H.clone()
    U = torch.empty((d, d), dtype=torch.float32, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    G.gptq_prepare_hinv(H, p, U, perm, dead, None, st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, 0]
    return p, H_copy, U, perm, dead


def _gpu_quantize(Wd, U, perm, dead, p, q):
    import post_weight_quantization_18_b200 as G
    n, d = Wd.shape
    Gn = 1 if q.group_size == -1 else d // q.group_size
    codes = torch.empty((n, d), dtype=torch.uint8, device="cuda")
    S = torch.empty((n, Gn), dtype=torch.float32, device="cuda")
    Z = torch.empty((n, Gn), dtype=torch.float32, device="cuda")
    gi = torch.empty(d, dtype=torch.int32, device="cuda")
    ws = torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    G.gptq_quantize_layer(Wd, U, perm, dead, p, codes, S, Z, gi, ws, st)
    qw = torch.empty((n, (d * q.bits + 31) // 32), dtype=torch.int32, device="cuda")
    s16 = torch.empty((n, Gn), dtype=torch.int16, device="cuda")
    z16 = torch.empty((n, Gn), dtype=torch.int16, device="cuda")
    G.gptq_pack(codes, q.bits, S, Z, qw, s16, z16)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, 0]
    return codes, S, Z, gi, qw, s16, z16


def _check_hessian_rows(H64, Hg, rows):
    got = Hg[rows].cpu().double().numpy()
    ref = H64[rows]
    up = np.arange(ref.shape[1])[None, :] >= rows[:, None]
    rel = np.linalg.norm((got - ref)[up]) / np.linalg.norm(ref[up])
    assert rel <= 1e-4, rel


def _U_times(U, E, rows=2048):
    """U^T (U E) in float64 for a few columns E, streaming the float32 U in row blocks."""
    d = U.shape[0]
    Ue = np.zeros((d, E.shape[1]))
    for r0 in range(0, d, rows):
        Ue[r0:r0 + rows] = U[r0:r0 + rows].astype(np.float64) @ E
    out = np.zeros_like(Ue)
    for r0 in range(0, d, rows):
        out += U[r0:r0 + rows].astype(np.float64).T @ Ue[r0:r0 + rows]
    return out


def _check_U(H64, Ug, perm, dead, lam, ks):
    """Componentwise backward error of H_d (U^T U e_k) = e_k in the permuted space, with
    H_d = H[pi][:, pi] + (dead + lambda) I from the oracle's H; the scale of each component is
    |H_d| |v|."""
    pi = perm.cpu().numpy().astype(np.int64)
    deadm = dead.cpu().numpy().astype(np.float64)
    E = np.zeros((Ug.shape[0], len(ks)))
    E[ks, np.arange(len(ks))] = 1.0
    Vp = _U_times(Ug, E)                    # v = H_d^-1 e_k (permuted coordinates)
    V = np.zeros_like(Vp)
    V[pi] = Vp                              # original channel order, as H has it
    HVp = (H64 @ V)[pi] + (deadm[:, None] + lam) * Vp
    scale = (np.abs(H64) @ np.abs(V))[pi] + (deadm[:, None] + lam) * np.abs(Vp)
    res = np.max(np.abs(HVp - E) / (scale + 1e-300))
    assert res <= 1e-4, res


def _check_U_tail(H64, Ug, perm, dead, lam, tail=1024):
    """The trailing block U[F, F], F = the last `tail` sweep positions, depends only on H_FF:
    it is the upper Cholesky factor of (H_FF + dead + lambda I)^-1. The oracle factors that
    block of its own H by the pages' three steps and compares entrywise."""
    d = Ug.shape[0]
    t = min(tail, d)
    pi = perm.cpu().numpy().astype(np.int64)[d - t:]
    HFF = H64[np.ix_(pi, pi)].copy()
    HFF += np.diag(dead.cpu().numpy()[d - t:].astype(np.float64) + lam)
    _, Uo = prep.upper_chol_of_inverse(HFF)
    Ut = Ug[d - t:, d - t:].astype(np.float64)
    rel = np.linalg.norm(Ut - Uo) / np.linalg.norm(Uo)
    assert rel <= 1e-4, rel


def _check_prepared(H64, Hg, U, perm, dead, q, act_order, rng, n_hrows, n_k):
    d = H64.shape[0]
    _check_hessian_rows(H64, Hg, np.sort(rng.choice(d, n_hrows, replace=False)))
    diag = np.diag(H64)
    pi = perm.cpu().numpy().astype(np.int64)
    if act_order:
        assert_valid_desc_order(pi, diag)
    dp = diag[pi]
    dp = np.where(dp == 0, 1.0, dp)
    lam = q.percdamp * dp.mean()
    Ug = U.cpu().numpy()
    _check_U(H64, Ug, perm, dead, lam, rng.choice(d, n_k, replace=False))
    _check_U_tail(H64, Ug, perm, dead, lam)
    return Ug


def _run_hessian_group(X, linears, q, rng, n_rows, n_hrows=16, n_k=4):
    """All checks for the linears that share calibration input X (see the module docstring)."""
    act_order = q.act_order
    Xd = X.cuda()
    p, Hg, U, perm, dead = _gpu_prepare(Xd, q, 1 if act_order else 0)
    del Xd
    H64 = hs.hessian(X, chunk=CHUNK)            # the oracle's H, from every token
    Ug = _check_prepared(H64, Hg, U, perm, dead, q, act_order, rng, n_hrows, n_k)
    del Hg
    d = H64.shape[0]
    samples = []
    for lin in linears:
        W = lin.make()
        rows = np.sort(rng.choice(W.shape[0], n_rows, replace=False))
        Wd = W.cuda()
        codes, S, Z, gi, qw, s16, z16 = _gpu_quantize(Wd, U, perm, dead, p, q)
        pi = perm.cpu().numpy().astype(np.int64)
        c = codes[rows].cpu().numpy()
        Sg, Zg = S[rows].cpu().double().numpy(), Z[rows].cpu().double().numpy()
        W64 = W[rows].double().numpy()
        tc = trajectory_check(W64, Ug, pi, dead.cpu().numpy(), c, Sg, Zg, q.bits, q.group_size,
                              q.sym)
        assert tc["bad_codes"] == 0 and tc["z_bad"] == 0 and tc["s_rel"] <= 1e-4, (lin.name, tc)
        g_idx = np.empty(d, np.int64)
        g_idx[pi] = (np.arange(d) // q.group_size) if q.group_size != -1 else 0
        assert np.array_equal(gi.cpu().numpy(), g_idx), lin.name
        ow, os16, oz16 = pk.pack(c, S[rows].cpu().numpy(), Z[rows].cpu().numpy(), q.bits)
        assert np.array_equal(qw[rows].cpu().numpy().view(np.uint32), ow), lin.name
        assert np.array_equal(s16[rows].cpu().numpy().view(np.uint16), os16), lin.name
        assert np.array_equal(z16[rows].cpu().numpy().view(np.uint16), oz16), lin.name
        samples.append(dict(name=lin.name, W=W, Wd=Wd, rows=rows, W64=W64,
                            res=dict(codes=c, S=Sg, Z=Zg, g_idx=gi.cpu().numpy().astype(np.int64))))
        del codes, S, Z, gi, qw, s16, z16
    del Ug
    # The oracle on the stacked sample rows of every linear of this Hessian.
    W64_all = np.concatenate([smp["W64"] for smp in samples])
    ora = oracle.gptq_layer(W64_all, H64, q.bits, q.group_size, q.sym, act_order=act_order)
    if act_order:
        # compare on the oracle's permutation: GPU prepare and sweep given pi_oracle
        H = torch.empty((d, d), dtype=torch.float32, device="cuda")
        import post_weight_quantization_18_b200 as G
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        Xd = X.cuda()
        G.gptq_hessian_accumulate(H, Xd, 2.0, False, st)
        del Xd
        p = G.make_params(q.bits, q.group_size, q.sym, 2, q.block_size, q.percdamp)
        perm = torch.as_tensor(ora["perm"], dtype=torch.int32).cuda()
        G.gptq_prepare_hinv(H, p, U, perm, dead, None, st)
        torch.cuda.synchronize()
        assert st.cpu().tolist() == [0, 0]
        del H
        for smp in samples:
            codes, S, Z, gi, *_ = _gpu_quantize(smp["Wd"], U, perm, dead, p, q)
            r = smp["rows"]
            smp["res"] = dict(codes=codes[r].cpu().numpy(), S=S[r].cpu().double().numpy(),
                              Z=Z[r].cpu().double().numpy(),
                              g_idx=gi.cpu().numpy().astype(np.int64))
    # Acceptance on the sampled rows of every linear (rows stacked as the oracle ran them).
    cat = lambda key: np.concatenate([smp["res"][key] for smp in samples])
    gpu = dict(codes=cat("codes"), S=cat("S"), Z=cat("Z"), perm=ora["perm"])
    ties = {r: (j, dist) for r, j, dist in first_divergence_ties(gpu, ora, q.bits, q.group_size,
                                                                 q.sym)}
    r0 = 0
    for smp in samples:
        k = len(smp["rows"])
        o = dict(codes=ora["codes"][r0:r0 + k], S=ora["S"][r0:r0 + k], Z=ora["Z"][r0:r0 + k],
                 g_idx=ora["g_idx"])
        res = smp["res"]
        agree = float(np.mean(res["codes"] == o["codes"]))
        e_g = er.layer_error(smp["W64"], er.dequant_matrix(res["codes"], res["S"], res["Z"],
                                                           res["g_idx"]), H64)
        e_o = er.layer_error(smp["W64"], er.dequant_matrix(o["codes"], o["S"], o["Z"],
                                                           o["g_idx"]), H64)
        mine = {r - r0: ties[r] for r in ties if r0 <= r < r0 + k}
        msg = (f"{smp['name']}: agree {agree:.6f}, error {e_g:.6e} vs oracle {e_o:.6e}, "
               f"first divergences (row: sweep position, distance to the boundary) {mine}")
        print(msg)
        assert abs(e_g - e_o) <= 1e-3 * e_o, msg
        if agree < 0.999:
            assert all(dist <= TIE_BAND for _, dist in mine.values()), msg
        r0 += k
        del smp["Wd"]
    # The sweep on the oracle's own U, order and dead columns (U rounded to fp32).
    import post_weight_quantization_18_b200 as G
    n_all = W64_all.shape[0]
    Wall = torch.cat([smp["W"][smp["rows"]] for smp in samples]).contiguous().cuda()
    Uo = torch.from_numpy(ora["U"].astype(np.float32)).cuda()
    del U
    po = torch.as_tensor(ora["perm"], dtype=torch.int32).cuda()
    do = torch.as_tensor(ora["dead"], dtype=torch.uint8).cuda()
    p = G.make_params(q.bits, q.group_size, q.sym, G.GPTQ_ORDER_GIVEN, q.block_size, q.percdamp)
    codes, *_ = _gpu_quantize(Wall, Uo, po, do, p, q)
    agree_sweep = float(np.mean(codes.cpu().numpy() == ora["codes"]))
    print(f"sweep on the oracle's U, {n_all} rows: agree {agree_sweep:.6f}")
    assert agree_sweep >= 0.999, agree_sweep
    del Uo, perm, dead, H64
    torch.cuda.empty_cache()


def test_full_tiny_256_identity_hessian_is_rtn():
    """The small fp32 workload at H = I: GPU GPTQ codes = GPU RTN codes = oracle RTN codes."""
    import post_weight_quantization_18_b200 as G
    wl = li.WORKLOADS["tiny_256"]
    lin, q = wl.linears[0], wl.quant
    W = lin.make()
    d = W.shape[1]
    out = G.quantize_layer(W.cuda(), H=torch.eye(d, device="cuda"), bits=q.bits,
                           group_size=q.group_size, sym=q.sym)
    codes_rtn, s_rtn, z_rtn = G.rtn(W.cuda(), q.bits, q.group_size, q.sym)
    ora = oracle.rtn_layer(W.numpy(), q.bits, q.group_size, q.sym)
    np.testing.assert_array_equal(out.codes.cpu().numpy(), codes_rtn.cpu().numpy())
    np.testing.assert_array_equal(codes_rtn.cpu().numpy(), ora["codes"])
    np.testing.assert_array_equal(s_rtn.cpu().numpy(), ora["S"])
    np.testing.assert_array_equal(z_rtn.cpu().numpy(), ora["Z"])


def test_full_llama7b_attn_proj():
    wl = li.WORKLOADS["llama7b_attn_proj"]
    _run_hessian_group(wl.acts[0].make(), wl.linears, wl.quant, np.random.default_rng(7),
                       n_rows=24, n_hrows=32, n_k=8)


def test_full_llama7b_mlp_act_order_3bit():
    wl = li.WORKLOADS["llama7b_mlp"]
    rng = np.random.default_rng(8)
    for act in wl.acts:        # gate and up share one Hessian; down has its own
        lins = [lin for lin in wl.linears if lin.act == act.name]
        _run_hessian_group(act.make(), lins, wl.quant, rng, n_rows=12 if len(lins) > 1 else 16)


def test_full_llama13b_block_shared_hessians():
    wl = li.WORKLOADS["llama13b_block"]
    rng = np.random.default_rng(9)
    for act in wl.acts:        # q/k/v share one Hessian, gate/up another
        lins = [lin for lin in wl.linears if lin.act == act.name]
        _run_hessian_group(act.make(), lins, wl.quant, rng, n_rows=8)


def test_full_llama70b_down_proj_per_row_symmetric():
    wl = li.WORKLOADS["llama70b_down_proj"]
    _run_hessian_group(wl.acts[0].make(), wl.linears, wl.quant, np.random.default_rng(10),
                       n_rows=8, n_hrows=8, n_k=3)
