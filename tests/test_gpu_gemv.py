"""GPU parity: the dequantizing matrix-vector product on packed layers against the oracle.

The kernel sums in fp32, so each output is compared with the float64 oracle within
1e-5 * sum_c |w_hat[r, c] x[c]| (a bound on fp32 summation error for these lengths)."""
import numpy as np
import pytest
import torch

from oracle import gemv as gv

pytestmark = pytest.mark.gpu


def _packed_layer(n, d, bits, g, seed, gidx_perm=False):
    import post_weight_quantization_18_b200 as G
    gen = torch.Generator().manual_seed(seed)
    codes = torch.randint(0, 2 ** bits, (n, d), generator=gen, dtype=torch.int32).to(torch.uint8)
    n_groups = 1 if g == -1 else d // g
    S = torch.rand((n, n_groups), generator=gen) * 0.02 + 0.001
    Z = torch.randint(0, 2 ** bits, (n, n_groups), generator=gen).float()
    qw = torch.empty((n, d * bits // 32), dtype=torch.int32, device="cuda")
    s16 = torch.empty((n, n_groups), dtype=torch.int16, device="cuda")
    z16 = torch.empty((n, n_groups), dtype=torch.int16, device="cuda")
    G.gptq_pack(codes.cuda(), bits, S.cuda(), Z.cuda(), qw, s16, z16)
    if gidx_perm:
        g_idx = torch.from_numpy(np.random.default_rng(seed).permutation(d) // g).to(torch.int32)
    else:
        g_idx = None
    return qw, s16, z16, g_idx, n_groups


def _check(qw, s16, z16, g_idx, d, bits, g, X):
    import post_weight_quantization_18_b200 as G
    n = qw.shape[0]
    Y = torch.full((X.shape[0], n), float("nan"), device="cuda")
    G.gptq_dequant_gemv(qw, d, bits, s16, z16, g, None if g_idx is None else g_idx.cuda(),
                        X.cuda(), Y)
    torch.cuda.synchronize()
    gi = (np.arange(d) // g if g > 0 else np.zeros(d, np.int64)) if g_idx is None else \
        g_idx.numpy()
    qn = qw.cpu().numpy().view(np.uint32)
    sn = s16.cpu().numpy().view(np.uint16)
    zn = z16.cpu().numpy().view(np.uint16)
    Xn = X.float().numpy().astype(np.float64)
    ref = gv.dequant_gemv(qn, sn, zn, gi, d, bits, Xn)
    bound = np.abs(Xn) @ np.abs(_w_hat(qn, sn, zn, gi, d, bits)).T
    err = np.abs(Y.cpu().numpy() - ref)
    assert np.all(np.isfinite(Y.cpu().numpy()))
    assert np.all(err <= 1e-5 * bound + 1e-6), float(np.max(err / (bound + 1e-30)))


def _w_hat(qn, sn, zn, gi, d, bits):
    from oracle import pack as pk
    codes = pk.unpack_rows(qn, d, bits).astype(np.float64)
    S, Z = gv.fp16_bits_to_f64(sn), gv.fp16_bits_to_f64(zn)
    return (codes - Z[:, gi]) * S[:, gi]


@pytest.mark.parametrize("n,d,bits,g,perm,batch", [
    (1000, 4096, 4, 128, False, 1),   # contiguous groups, ragged row count
    (512, 2048, 3, 128, True, 4),     # act-order g_idx, 3-bit words straddling
    (256, 1024, 2, -1, False, 2),     # one group per row
    (384, 2048, 8, 32, False, 8),     # 8-bit, batch 8
    (300, 1024, 4, 16, False, 1),     # groups shorter than a 32-column run
    # tensor-core path: groups of whole 128-column chunks, d_in a multiple of 128
    (1000, 4096, 4, 256, False, 3),   # ragged last 16-row tile, groups over two chunks
    (70, 128, 4, 128, False, 1),      # one chunk per row, fewer chunks than warps
    (384, 2048, 8, 128, False, 8),    # 8-bit, full batch
    (136, 3072, 2, 128, False, 5),    # 2-bit, odd batch
    (64, 1152, 4, -1, False, 1),      # one group per row, chunk count not a multiple of warps
    (96, 1056, 4, -1, False, 2),      # d_in not a multiple of 128: warp-per-row path
    # 3-bit codes on the tensor cores: runs of 3 words, pairs straddling word boundaries
    (1000, 4096, 3, 128, False, 1),
    (136, 3072, 3, -1, False, 5),
    (40, 2048, 3, 256, False, 8),     # fewer rows than one CTA's tiles
    (520, 1024, 2, 128, False, 1),    # 2-bit, ragged last tile
])
def test_dequant_gemv_matches_oracle(n, d, bits, g, perm, batch):
    qw, s16, z16, g_idx, _ = _packed_layer(n, d, bits, g, seed=n + d + bits, gidx_perm=perm)
    X = torch.randn((batch, d), generator=torch.Generator().manual_seed(d)).half()
    _check(qw, s16, z16, g_idx, d, bits, g, X)


def test_dequant_gemv_on_a_gptq_layer():
    """End to end: GPTQ on the GPU, packed by gptq_pack, consumed by the GEMV."""
    import post_weight_quantization_18_b200 as G
    from gpu_util import make_inputs
    W, X = make_inputs(256, 1024, 4000, seed=41)
    out = G.quantize_layer(W.cuda(), X=X.cuda(), bits=4, group_size=128, act_order=True)
    qw, s16, z16 = out.pack()
    xv = torch.randn((1, 1024), generator=torch.Generator().manual_seed(5)).half()
    _check(qw, s16, z16, out.g_idx.cpu(), 1024, 4, 128, xv)
