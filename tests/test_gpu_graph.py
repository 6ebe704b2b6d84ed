"""The C ABI calls recorded into a CUDA graph and replayed give the results of direct calls.

Every entry point only enqueues work on the caller's stream (no allocation, no host
synchronisation), so a caller may record a whole layer into a CUDA graph and replay it. Checked
here on the layer shapes the tests use: prepare, sweep and pack are deterministic, so a replay
from the same H must match the direct calls bit for bit; the Hessian kernel splits long token
ranges over CTAs that add into H, so its replay is compared within float rounding.
"""
import numpy as np
import pytest
import torch

from gpu_util import make_inputs

pytestmark = pytest.mark.gpu


def _buffers(n, d, p, bits, G_n):
    import post_weight_quantization_18_b200 as G
    dev = "cuda"
    return dict(
        U=torch.full((d, d), float("nan"), device=dev),
        perm=torch.full((d,), -1, dtype=torch.int32, device=dev),
        dead=torch.full((d,), 7, dtype=torch.uint8, device=dev),
        codes=torch.full((n, d), 255, dtype=torch.uint8, device=dev),
        scales=torch.full((n, G_n), float("nan"), device=dev),
        zeros=torch.full((n, G_n), float("nan"), device=dev),
        g_idx=torch.full((d,), -1, dtype=torch.int32, device=dev),
        ws=torch.empty(G.gptq_workspace_size(n, d, p), dtype=torch.uint8, device=dev),
        qweight=torch.zeros((n, (d * bits + 31) // 32), dtype=torch.int32, device=dev),
        s16=torch.zeros((n, G_n), dtype=torch.int16, device=dev),
        z16=torch.zeros((n, G_n), dtype=torch.int16, device=dev),
        status=torch.zeros(2, dtype=torch.int32, device=dev))


def _layer_calls(G, H, W, p, bits, b):
    G.gptq_prepare_hinv(H, p, b["U"], b["perm"], b["dead"], b["ws"], b["status"])
    G.gptq_quantize_layer(W, b["U"], b["perm"], b["dead"], p, b["codes"], b["scales"],
                          b["zeros"], b["g_idx"], b["ws"], b["status"])
    G.gptq_pack(b["codes"], bits, b["scales"], b["zeros"], b["qweight"], b["s16"], b["z16"])


@pytest.mark.parametrize("n,d,N,bits,g,sym,order", [
    (384, 1152, 6000, 4, 128, False, 0),     # several U recursion levels, ragged token count
    (256, 640, 3000, 3, 128, False, 1),      # act-order, 3-bit
    (128, 896, 2000, 4, -1, True, 0),        # per-row symmetric
])
def test_graph_replay_matches_direct_calls(n, d, N, bits, g, sym, order):
    import post_weight_quantization_18_b200 as G
    W, X = make_inputs(n, d, N, seed=9100 + d)
    Wd, Xd = W.cuda(), X.cuda()
    p = G.make_params(bits, g, sym, order)
    G_n = 1 if g == -1 else d // g

    H0 = torch.empty((d, d), device="cuda")
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    G.gptq_hessian_accumulate(H0, Xd, 2.0, False, st)

    # Direct calls.
    direct = _buffers(n, d, p, bits, G_n)
    H = H0.clone()
    _layer_calls(G, H, Wd, p, bits, direct)
    torch.cuda.synchronize()
    assert direct["status"].cpu().tolist() == [0, 0]

    # The same calls recorded once and replayed twice; H is refreshed inside the graph because
    # prepare overwrites it.
    rep = _buffers(n, d, p, bits, G_n)
    Hg = torch.empty_like(H0)
    Hx = torch.full((d, d), float("nan"), device="cuda")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        G.gptq_hessian_accumulate(Hx, Xd, 2.0, False, rep["status"])
        Hg.copy_(H0)
        _layer_calls(G, Hg, Wd, p, bits, rep)
    for _ in range(2):
        graph.replay()
        torch.cuda.synchronize()
        assert rep["status"].cpu().tolist() == [0, 0]
        for k in ("U", "perm", "dead", "codes", "scales", "zeros", "g_idx", "qweight", "s16",
                  "z16"):
            np.testing.assert_array_equal(rep[k].cpu().numpy(), direct[k].cpu().numpy(),
                                          err_msg=k)
        iu = np.triu_indices(d)
        h_rep, h_dir = Hx.cpu().numpy()[iu], H0.cpu().numpy()[iu]
        rel = np.linalg.norm(h_rep - h_dir) / np.linalg.norm(h_dir)
        assert rel <= 1e-6, rel
    del graph


def test_bench_counts_kernel_launches_from_recorded_graphs():
    """bench.py reports the kernels a step launches as the kernel nodes of the CUDA graphs it
    records from the C ABI calls; the count is positive and the same for two recordings."""
    import bench
    import post_weight_quantization_18_b200 as G
    from gpu_util import make_inputs
    W, X = make_inputs(64, 512, 4096, seed=5)
    Wd, Xd = W.cuda(), X.cuda()
    G.quantize_layer(Wd, X=Xd)              # first call: stream and attribute set-up
    torch.cuda.synchronize()
    counts = []
    for _ in range(2):
        gr, kept = bench.new_graph()
        with torch.cuda.graph(gr):
            G.quantize_layer(Wd, X=Xd, check=False)
        counts.append(bench.graph_kernel_nodes(gr) if kept else None)
    assert counts[0] is not None and counts[0] > 5 and counts[0] == counts[1], counts
