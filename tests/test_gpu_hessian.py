"""GPU parity: gptq_hessian_accumulate (tcgen05 bf16 SYRK, fp32 path) against the oracle."""
import numpy as np
import pytest
import torch

from gpu_util import f64, make_inputs
from oracle import hessian as hs

pytestmark = pytest.mark.gpu

RTOL_FRO = 1e-4  # relative Frobenius error bound on H


def _upper(a):
    return np.triu(a)


def _rel_fro(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("d,N", [(64, 64), (200, 1000), (256, 2048), (520, 3001), (1000, 777),
                                 (1536, 20000)])
def test_syrk_bf16_matches_oracle(d, N):
    import post_weight_quantization_18_b200 as G
    _, X = make_inputs(8, d, N, seed=100 + d)
    H = torch.full((d, d), 12345.0, dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(H, X.cuda(), 2.0, False)
    Hg = H.cpu().numpy().astype(np.float64)
    Ho = hs.hessian(f64(X))
    assert _rel_fro(_upper(Hg), _upper(Ho)) <= RTOL_FRO
    # the strictly lower triangle is neither read nor written
    low = np.tril_indices(d, -1)
    assert np.all(Hg[low] == 12345.0)
    # diagonal: every entry, not just the norm
    np.testing.assert_allclose(np.diag(Hg), np.diag(Ho), rtol=1e-4)


def test_syrk_accumulate_chunks_and_padded_ld():
    """H from two token chunks with accumulate=1 equals H of the whole; X with ldx > d_in."""
    import post_weight_quantization_18_b200 as G
    d, N = 384, 5000
    _, X = make_inputs(8, d, N, seed=7)
    Xp = torch.zeros((N, d + 24), dtype=torch.bfloat16)
    Xp[:, :d] = X
    Xd = Xp.cuda()[:, :d]
    H = torch.zeros((d, d + 4), dtype=torch.float32, device="cuda")[:, :d]
    G.gptq_hessian_accumulate(H, Xd[:3000], 2.0, False)
    G.gptq_hessian_accumulate(H, Xd[3000:], 2.0, True)
    Hg = H.cpu().numpy().astype(np.float64)
    assert _rel_fro(_upper(Hg), _upper(hs.hessian(f64(X)))) <= RTOL_FRO


def test_syrk_zero_tokens():
    import post_weight_quantization_18_b200 as G
    d = 128
    H = torch.full((d, d), 5.0, device="cuda")
    X = torch.zeros((0, d), dtype=torch.bfloat16, device="cuda")
    G.gptq_hessian_accumulate(H, X, 2.0, False)
    Hg = H.cpu().numpy()
    assert np.all(np.triu(Hg) == 0) and np.all(Hg[np.tril_indices(d, -1)] == 5.0)


def test_syrk_fp32_input():
    import post_weight_quantization_18_b200 as G
    _, X = make_inputs(8, 256, 2048, seed=1001, x_dtype=torch.float32, chan_sigma=0.5,
                       outlier_frac=0.0)
    H = torch.empty((256, 256), device="cuda")
    G.gptq_hessian_accumulate(H, X.cuda(), 2.0, False)
    Hg = H.cpu().numpy().astype(np.float64)
    Ho = hs.hessian(f64(X))
    assert _rel_fro(_upper(Hg), _upper(Ho)) <= RTOL_FRO
    np.testing.assert_allclose(np.diag(Hg), np.diag(Ho), rtol=5e-5)


def test_syrk_rejects_misaligned_ld():
    import post_weight_quantization_18_b200 as G
    X = torch.zeros((16, 130), dtype=torch.bfloat16, device="cuda")
    H = torch.zeros((130, 130), device="cuda")
    with pytest.raises(G.GPTQError):
        G.gptq_hessian_accumulate(H, X, 2.0, False)   # ldx = 130 is not a multiple of 8
