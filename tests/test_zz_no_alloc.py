"""gptq_quantize_layer_noalloc — the variant for callers that cannot allocate device memory
(for example a plugin inside another runtime that owns all device memory, or a service that must
not allocate once it is serving): it uses a fixed scratch array compiled into the library instead
of a caller-provided workspace.

Checked through the C ABI against gptq_quantize_layer on the same inputs, on two calls in a row
(the second call finds the first call's data still in the shared array), with the same
tolerances as the other sweep tests. Also checks that a layer too large for the array is
rejected on the host. Collected last so that a failure here stops a -x run only after every
other test has run.
"""
import numpy as np
import pytest
import torch

from gpu_util import make_inputs

pytestmark = pytest.mark.gpu


def _prepared(n, d, N, seed, bits, g, sym, order):
    import post_weight_quantization_18_b200 as G
    W, X = make_inputs(n, d, N, seed=seed)
    Wd, Xd = W.cuda(), X.cuda()
    p = G.make_params(bits, g, sym, order)
    H = torch.empty((d, d), dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(H, Xd, 2.0, False)
    U = torch.empty((d, d), dtype=torch.float32, device="cuda")
    perm = torch.empty(d, dtype=torch.int32, device="cuda")
    dead = torch.empty(d, dtype=torch.uint8, device="cuda")
    G.gptq_prepare_hinv(H, p, U, perm, dead)
    return Wd, U, perm, dead, p


def _outputs(n, d, g):
    G_n = 1 if g == -1 else d // g
    return (torch.full((n, d), 255, dtype=torch.uint8, device="cuda"),
            torch.full((n, G_n), float("nan"), device="cuda"),
            torch.full((n, G_n), float("nan"), device="cuda"),
            torch.full((d,), -1, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("bits,g,sym,order", [(4, 128, False, 0), (3, 128, False, 1),
                                              (4, -1, True, 0)])
def test_noalloc_matches_workspace_entry_point(bits, g, sym, order):
    import post_weight_quantization_18_b200 as G
    n, d, N = 256, 512, 8000
    W, U, perm, dead, p = _prepared(n, d, N, 11 + bits + order, bits, g, sym, order)
    ref = _outputs(n, d, g)
    ws = torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    G.gptq_quantize_layer(W, U, perm, dead, p, *ref, ws, st)
    for call in range(2):
        out = _outputs(n, d, g)
        st2 = torch.zeros(2, dtype=torch.int32, device="cuda")
        G.gptq_quantize_layer_noalloc(W, U, perm, dead, p, *out, st2)
        torch.cuda.synchronize()
        assert st.cpu().tolist() == [0, 0] and st2.cpu().tolist() == [0, 0]
        codes_r, codes_o = ref[0].cpu().numpy(), out[0].cpu().numpy()
        agree = float(np.mean(codes_r == codes_o))
        assert agree >= 0.999, (call, agree)
        s_r, s_o = ref[1].cpu().numpy(), out[1].cpu().numpy()
        assert np.all(np.isfinite(s_o))
        np.testing.assert_allclose(s_o, s_r, rtol=1e-4)
        np.testing.assert_allclose(out[2].cpu().numpy(), ref[2].cpu().numpy(), atol=0.5)
        np.testing.assert_array_equal(out[3].cpu().numpy(), ref[3].cpu().numpy())


def test_noalloc_rejects_layer_larger_than_scratch():
    import post_weight_quantization_18_b200 as G
    n, d = 4096, 4096   # 128 MiB of scratch needed, more than GPTQ_NOALLOC_SCRATCH_BYTES
    p = G.make_params(4, 128)
    assert G.gptq_workspace_size(n, d, p) > G.GPTQ_NOALLOC_SCRATCH_BYTES
    W = torch.zeros((n, d), dtype=torch.bfloat16, device="cuda")
    U = torch.zeros((d, d), device="cuda")
    perm = torch.arange(d, dtype=torch.int32, device="cuda")
    dead = torch.zeros(d, dtype=torch.uint8, device="cuda")
    out = _outputs(n, d, 128)
    with pytest.raises(G.GPTQError) as e:
        G.gptq_quantize_layer_noalloc(W, U, perm, dead, p, *out)
    assert e.value.code == 3  # GPTQ_ERR_WORKSPACE
