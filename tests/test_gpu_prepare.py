"""GPU parity: gptq_prepare_hinv against the oracle's three-step route."""
import numpy as np
import pytest
import torch

from gpu_util import assert_valid_desc_order, f64, make_inputs
from oracle import hessian as hs
from oracle import prepare as prep

pytestmark = pytest.mark.gpu


def _run(H64, order=0, perm=None, percdamp=0.01):
    import post_weight_quantization_18_b200 as G
    d = H64.shape[0]
    H = torch.tensor(np.triu(H64), dtype=torch.float32, device="cuda")
    U = torch.empty((d, d), device="cuda")
    p = torch.tensor(perm, dtype=torch.int32, device="cuda") if perm is not None else \
        torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    G.gptq_prepare_hinv(H, G.make_params(order=order, percdamp=percdamp), U, p, dead, None, st)
    torch.cuda.synchronize()
    return (U.cpu().numpy().astype(np.float64), p.cpu().numpy(), dead.cpu().numpy(),
            st.cpu().numpy())


@pytest.mark.parametrize("d,N,half", [(100, 2000, False), (256, 4096, False), (300, 3000, True),
                                      (640, 8000, False), (1000, 12000, True)])
def test_U_matches_oracle(d, N, half):
    _, X = make_inputs(4, d, N, seed=200 + d, half_normal=half)
    H64 = hs.hessian(f64(X))
    U, perm, dead, st = _run(H64)
    assert st[0] == 0
    assert np.array_equal(perm, np.arange(d)) and not dead.any()
    Uo = prep.prepare(H64, np.zeros((1, d)), 0.01)["U"]
    assert np.all(U[np.tril_indices(d, -1)] == 0)
    rel = np.linalg.norm(U - Uo) / np.linalg.norm(Uo)
    assert rel <= 1e-4, rel
    # the defining identity in fp64 from the GPU's U
    Hd, _ = prep.damp(H64, 0.01)
    assert np.abs(U.T @ U @ Hd - np.eye(d)).max() <= 1e-3


def test_act_order_and_given_perm():
    d = 384
    _, X = make_inputs(4, d, 6000, seed=31)
    H64 = hs.hessian(f64(X))
    U, perm, dead, st = _run(H64, order=1)
    assert st[0] == 0
    assert_valid_desc_order(perm, np.diag(H64))
    ora = prep.prepare(H64, np.zeros((1, d)), 0.01, act_order=True)
    U2, perm2, _, st2 = _run(H64, order=2, perm=ora["perm"])
    assert st2[0] == 0 and np.array_equal(perm2, ora["perm"])
    assert np.linalg.norm(U2 - ora["U"]) / np.linalg.norm(ora["U"]) <= 1e-4
    if np.array_equal(perm, ora["perm"]):
        assert np.linalg.norm(U - ora["U"]) / np.linalg.norm(ora["U"]) <= 1e-4


def test_dead_columns():
    d = 256
    _, X = make_inputs(4, d, 3000, seed=41)
    Xn = f64(X)
    Xn[:, [3, 130, 255]] = 0
    H64 = hs.hessian(Xn)
    U, perm, dead, st = _run(H64)
    assert st[0] == 0
    assert np.flatnonzero(dead).tolist() == [3, 130, 255]
    Uo = prep.prepare(H64, np.zeros((1, d)), 0.01)["U"]
    assert np.linalg.norm(U - Uo) / np.linalg.norm(Uo) <= 1e-4


def test_not_spd_is_reported_not_trapped():
    """percdamp = 0 on an indefinite matrix: the device status says NOT_SPD; no hang, no trap."""
    d = 200
    H = -np.eye(d)
    U, perm, dead, st = _run(H, percdamp=0.0)
    assert st[0] == 16  # GPTQ_ERR_NOT_SPD
    assert 0 <= st[1] < d


def test_nonfinite_is_reported():
    d = 128
    H = np.eye(d)
    H[5, 5] = np.nan
    U, perm, dead, st = _run(H)
    assert st[0] in (16, 17)
