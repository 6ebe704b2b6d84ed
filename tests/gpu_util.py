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
                 perm=None, percdamp=0.01):
    """Hessian -> prepare -> sweep on the GPU. Returns host numpy arrays."""
    import post_weight_quantization_18_b200 as G
    Wd = W.cuda()
    Hd = None
    if H is not None:
        Hd = torch.as_tensor(H, dtype=torch.float32).cuda().contiguous()
    Xd = X.cuda() if X is not None else None
    pd = torch.as_tensor(perm, dtype=torch.int32).cuda() if perm is not None else None
    out = G.quantize_layer(Wd, X=Xd, H=Hd, bits=bits, group_size=group_size, sym=sym,
                           act_order=act_order, perm=pd, percdamp=percdamp)
    torch.cuda.synchronize()
    return dict(codes=out.codes.cpu().numpy(), S=out.scales.cpu().numpy().astype(np.float64),
                Z=out.zeros.cpu().numpy().astype(np.float64),
                g_idx=out.g_idx.cpu().numpy().astype(np.int64),
                perm=out.perm.cpu().numpy().astype(np.int64), dead=out.dead.cpu().numpy())


def layer_err(W64, res, H64):
    return er.layer_error(W64, er.dequant_matrix(res["codes"], res["S"], res["Z"], res["g_idx"]),
                          H64)


def compare_with_oracle(W, X, bits=4, group_size=128, sym=False, act_order=False,
                        given_perm=False, code_agree=0.999, err_rtol=1e-3):
    """Full GPU pipeline vs the oracle on the same seeded inputs. Returns (agree, rel_err)."""
    W64, X64 = f64(W), f64(X)
    H64 = hs.hessian(X64)
    ora = oracle.gptq_layer(W64, H64, bits, group_size, sym, act_order=act_order)
    perm = ora["perm"] if given_perm else None
    gpu = gpu_pipeline(W, X, bits=bits, group_size=group_size, sym=sym,
                       act_order=act_order and not given_perm, perm=perm)
    if act_order and not given_perm:
        assert_valid_desc_order(gpu["perm"], np.diag(H64))
    agree = float(np.mean(gpu["codes"] == ora["codes"]))
    e_gpu, e_ora = layer_err(W64, gpu, H64), layer_err(W64, ora, H64)
    rel = abs(e_gpu - e_ora) / e_ora
    assert agree >= code_agree, f"code agreement {agree:.6f}"
    assert rel <= err_rtol, f"error {e_gpu} vs oracle {e_ora} (rel {rel:.2e})"
    assert np.all(gpu["codes"] < 2 ** bits)
    return agree, rel, gpu, ora


def assert_valid_desc_order(perm, diag, rtol=1e-5):
    """perm must be a permutation sorting diag descending, up to near-ties (fp32 vs fp64 H)."""
    assert sorted(perm.tolist()) == list(range(len(diag)))
    v = diag[perm]
    bad = v[1:] > v[:-1] * (1 + rtol) + 1e-30
    assert not np.any(bad), f"{int(bad.sum())} out-of-order pairs"
