"""GPU parity of the product kernel (gptq_gemm_f32) against float64 products.

Bound (componentwise): |C_gpu - C_64| <= tol * (|alpha| (|A| |B|)_mn + |beta| |C_mn|) with
tol = 1e-4. Each product carries the three-term TF32 split error (about 2^-21 relative: the
hi*lo terms lose the low bits of the lo parts and lo*lo is dropped); the tensor core adds into
its fp32 accumulator with truncation, at most one ulp per accumulate step, over at most 384
steps per accumulator (three MMAs per 8-wide k step, K <= 1024 per accumulator) before the
stretch is added into C in fp32 round-to-nearest: 384 * 2^-23 = 4.6e-5 of the sum of |terms|.
The CUDA-core kernels (products up to 512^3) are well inside the same bound.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL = 1e-4


def _run(M, N, K, ta, tb, alpha, beta, seed, scale_a=1.0):
    import post_weight_quantization_18_b200 as G
    g = torch.Generator().manual_seed(seed)
    A = (torch.randn((K, M) if ta else (M, K), generator=g) * scale_a).float()
    B = torch.randn((N, K) if tb else (K, N), generator=g).float()
    C = torch.randn((M, N), generator=g).float()
    Cd = C.cuda()
    G.gptq_gemm_f32(A.cuda(), B.cuda(), Cd, alpha=alpha, beta=beta, trans_a=ta, trans_b=tb)
    torch.cuda.synchronize()
    A64 = A.double().numpy()
    B64 = B.double().numpy()
    opA = A64.T if ta else A64
    opB = B64.T if tb else B64
    ref = alpha * (opA @ opB) + beta * C.double().numpy()
    scale = abs(alpha) * (np.abs(opA) @ np.abs(opB)) + abs(beta) * np.abs(C.double().numpy())
    err = np.abs(Cd.cpu().double().numpy() - ref)
    return float(np.max(err / (scale + 1e-300)))


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (300, 200, 77), (1000, 1000, 1000),
                                   (2048, 1536, 3000), (129, 4097, 2049)])
@pytest.mark.parametrize("ta,tb", [(False, False), (True, False), (False, True)])
def test_gemm_matches_float64(M, N, K, ta, tb):
    assert _run(M, N, K, ta, tb, -1.0, 1.0, seed=M + N + K) <= TOL


def test_gemm_beta_zero_and_scaling():
    assert _run(640, 768, 1024, False, False, 0.5, 0.0, seed=3, scale_a=1e-3) <= TOL


def test_gemm_large_tensor_core_product():
    """A product of the lazy-update shape class on the tcgen05 path: 4096 x 4096 x 4096, each
    operand 64 MB (the three together are larger than L2)."""
    assert _run(4096, 4096, 4096, False, False, -1.0, 1.0, seed=11) <= TOL
