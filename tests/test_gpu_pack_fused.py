"""GPU parity of the fused sweep-and-pack entry point (gptq_quantize_pack_layer): on the same
U, order and dead columns it writes exactly the words and fp16 parameters that
gptq_quantize_layer followed by gptq_pack writes, bit for bit, and the same fp32 parameters and
g_idx. The packing itself is pinned against the oracle's packing by tests/test_gpu_sweep.py."""
import numpy as np
import pytest
import torch

from gpu_util import make_inputs
from oracle import pack as pk

pytestmark = pytest.mark.gpu


def _prepared(G, X, p):
    d = X.shape[1]
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    H = torch.empty((d, d), device="cuda")
    G.gptq_hessian_accumulate(H, X.cuda(), 2.0, False, st)
    U = torch.empty((d, d), device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    G.gptq_prepare_hinv(H, p, U, perm, dead, None, st)
    return U, perm, dead, st


@pytest.mark.parametrize("n,d,bits,g,sym,order,static", [
    (300, 640, 4, 128, False, 0, False),      # several blocks, ragged rows
    (37, 256, 3, 128, False, 0, False),       # fewer rows than one sweep CTA
    (2100, 512, 4, 128, False, 0, False),     # two row panels
    (160, 1024, 4, -1, True, 0, False),       # one symmetric scale per row
    (96, 1280, 2, 64, False, 0, False),
    (64, 384, 8, 32, True, 0, False),
    (200, 512, 3, 128, False, 1, False),      # act-order: unpermute and pack in one kernel
    (1030, 384, 4, 128, False, 1, False),     # act-order, two panels
    (160, 512, 4, 128, False, 1, True),       # static groups with act-order
])
def test_fused_pack_equals_sweep_then_pack(n, d, bits, g, sym, order, static):
    import post_weight_quantization_18_b200 as G
    W, X = make_inputs(n, d, 4000, seed=n + d + bits)
    Wd = W.cuda()
    p = G.make_params(bits, g, sym, order, 128, 0.01, static)
    U, perm, dead, st = _prepared(G, X, p)
    Gn = 1 if g == -1 else d // g
    ws = torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device="cuda")
    # reference: sweep to codes, then pack
    codes = torch.empty((n, d), dtype=torch.uint8, device="cuda")
    S1 = torch.empty((n, Gn), device="cuda")
    Z1 = torch.empty((n, Gn), device="cuda")
    g1 = torch.empty(d, dtype=torch.int32, device="cuda")
    G.gptq_quantize_layer(Wd, U, perm, dead, p, codes, S1, Z1, g1, ws, st)
    q1 = torch.empty((n, d * bits // 32), dtype=torch.int32, device="cuda")
    s1 = torch.empty((n, Gn), dtype=torch.int16, device="cuda")
    z1 = torch.empty((n, Gn), dtype=torch.int16, device="cuda")
    G.gptq_pack(codes, bits, S1, Z1, q1, s1, z1)
    # fused
    q2 = torch.full((n, d * bits // 32), -1, dtype=torch.int32, device="cuda")
    s2 = torch.full((n, Gn), -1, dtype=torch.int16, device="cuda")
    z2 = torch.full((n, Gn), -1, dtype=torch.int16, device="cuda")
    S2 = torch.empty((n, Gn), device="cuda")
    Z2 = torch.empty((n, Gn), device="cuda")
    g2 = torch.empty(d, dtype=torch.int32, device="cuda")
    G.gptq_quantize_pack_layer(Wd, U, perm, dead, p, q2, s2, z2, S2, Z2, g2, ws, st)
    torch.cuda.synchronize()
    assert st.cpu().tolist() == [0, 0]
    np.testing.assert_array_equal(q2.cpu().numpy(), q1.cpu().numpy())
    np.testing.assert_array_equal(s2.cpu().numpy(), s1.cpu().numpy())
    np.testing.assert_array_equal(z2.cpu().numpy(), z1.cpu().numpy())
    np.testing.assert_array_equal(S2.cpu().numpy(), S1.cpu().numpy())
    np.testing.assert_array_equal(Z2.cpu().numpy(), Z1.cpu().numpy())
    np.testing.assert_array_equal(g2.cpu().numpy(), g1.cpu().numpy())
    # and the words are the oracle's packing of the codes
    ow, os16, oz16 = pk.pack(codes.cpu().numpy(), S1.cpu().numpy(), Z1.cpu().numpy(), bits)
    np.testing.assert_array_equal(q2.cpu().numpy().view(np.uint32), ow)
    np.testing.assert_array_equal(s2.cpu().numpy().view(np.uint16), os16)
