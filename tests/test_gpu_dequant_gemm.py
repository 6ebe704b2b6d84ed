"""GPU parity: the dequantizing GEMM (prefill batches) on packed 4-bit layers against the oracle.

The kernel multiplies activations by the codes exactly and sums in fp32, so each output is
compared with the float64 oracle within 1e-5 * sum_c |w_hat[r, c] x[c]| (a bound on fp32
summation error for these lengths), as the GEMV is."""
import numpy as np
import pytest
import torch

from oracle import gemv as gv

pytestmark = pytest.mark.gpu


def _packed_layer(n, d, g, seed):
    import post_weight_quantization_18_b200 as G
    gen = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 16, (n, d), generator=gen, dtype=torch.int32).to(torch.uint8)
    n_groups = 1 if g == -1 else d // g
    S = torch.rand((n, n_groups), generator=gen) * 0.02 + 0.001
    Z = torch.randint(0, 16, (n, n_groups), generator=gen).float()
    qw = torch.empty((n, d // 8), dtype=torch.int32, device="cuda")
    s16 = torch.empty((n, n_groups), dtype=torch.int16, device="cuda")
    z16 = torch.empty((n, n_groups), dtype=torch.int16, device="cuda")
    G.gptq_pack(codes.cuda(), 4, S.cuda(), Z.cuda(), qw, s16, z16)
    return qw, s16, z16


def _oracle(qw, s16, z16, d, g, X):
    from oracle import pack as pk
    qn = qw.cpu().numpy().view(np.uint32)
    sn = s16.cpu().numpy().view(np.uint16)
    zn = z16.cpu().numpy().view(np.uint16)
    gi = np.arange(d) // g if g > 0 else np.zeros(d, np.int64)
    Xn = X.float().numpy().astype(np.float64)
    ref = gv.dequant_gemv(qn, sn, zn, gi, d, 4, Xn)
    codes = pk.unpack_rows(qn, d, 4).astype(np.float64)
    S, Z = gv.fp16_bits_to_f64(sn), gv.fp16_bits_to_f64(zn)
    bound = np.abs(Xn) @ np.abs((codes - Z[:, gi]) * S[:, gi]).T
    return ref, bound


@pytest.mark.parametrize("n,d,g,m", [
    (256, 1024, 128, 128),    # one tile row of activations, two of weights
    (1000, 2048, 128, 300),   # ragged in both output dimensions
    (300, 4096, 256, 17),     # groups over two 128-column folds, few activation rows
    (136, 1152, -1, 260),     # one group per row, K not a multiple of 256
    (64, 128, 128, 1),        # a single fold, a single activation row
])
def test_dequant_gemm_matches_oracle(n, d, g, m):
    import post_weight_quantization_18_b200 as G
    qw, s16, z16 = _packed_layer(n, d, g, seed=n + d + m)
    X = torch.randn((m, d), generator=torch.Generator().manual_seed(m + d)).half()
    Y = torch.full((m, n), float("nan"), device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    G.gptq_dequant_gemm(qw, d, s16, z16, g, X.cuda(), Y, dev_status=st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, 0]
    ref, bound = _oracle(qw, s16, z16, d, g, X)
    out = Y.cpu().numpy()
    assert np.all(np.isfinite(out))
    err = np.abs(out - ref)
    assert np.all(err <= 1e-5 * bound + 1e-6), float(np.max(err / (bound + 1e-30)))


def test_dequant_gemm_agrees_with_gemv_and_repeats():
    """The GEMM at a batch the GEMV also takes gives the same products within the same bound,
    and two calls give bitwise the same Y (no atomics in the GEMM)."""
    import post_weight_quantization_18_b200 as G
    n, d, g = 512, 2048, 128
    qw, s16, z16 = _packed_layer(n, d, g, seed=7)
    X = torch.randn((8, d), generator=torch.Generator().manual_seed(3)).half().cuda()
    Y1 = torch.empty((8, n), device="cuda")
    Y2 = torch.empty((8, n), device="cuda")
    Yv = torch.empty((8, n), device="cuda")
    G.gptq_dequant_gemm(qw, d, s16, z16, g, X, Y1)
    G.gptq_dequant_gemm(qw, d, s16, z16, g, X, Y2)
    G.gptq_dequant_gemv(qw, d, 4, s16, z16, g, None, X, Yv)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)
    _, bound = _oracle(qw, s16, z16, d, g, X.cpu())
    assert np.all(np.abs(Y1.cpu().numpy() - Yv.cpu().numpy()) <= 2e-5 * bound + 2e-6)


def test_dequant_gemm_skips_when_status_is_set():
    """A status that already holds an error makes the call skip its work: Y keeps its contents."""
    import post_weight_quantization_18_b200 as G
    n, d, g = 128, 256, 128
    qw, s16, z16 = _packed_layer(n, d, g, seed=11)
    X = torch.randn((16, d)).half().cuda()
    Y = torch.full((16, n), 123.0, device="cuda")
    st = torch.tensor([16, 0], dtype=torch.int32, device="cuda")
    G.gptq_dequant_gemm(qw, d, s16, z16, g, X, Y, dev_status=st)
    torch.cuda.synchronize()
    assert torch.all(Y == 123.0)
