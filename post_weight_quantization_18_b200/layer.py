"""One-call convenience API over the C ABI: allocate outputs with torch, call the entry points.

    out = quantize_layer(W, X=X_tm, bits=4, group_size=128)          # H from calibration X
    out = quantize_layer(W, H=H, bits=3, act_order=True)             # H already accumulated

All arithmetic runs in the library's kernels; this module only sizes and allocates buffers,
orders the calls on the current stream and reads the device status word at the end.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib as L


@dataclass
class QuantizedLayer:
    codes: torch.Tensor        # uint8 [d_out, d_in], original column order
    scales: torch.Tensor       # fp32 [d_out, n_groups], sweep-group order
    zeros: torch.Tensor        # fp32 [d_out, n_groups]
    g_idx: torch.Tensor        # int32 [d_in]
    perm: torch.Tensor         # int32 [d_in]
    dead: torch.Tensor         # uint8 [d_in], sweep order
    bits: int
    group_size: int

    def pack(self):
        """(qweight int32 [d_out, ceil(d_in*bits/32)], scales fp16, zeros fp16)."""
        n, d = self.codes.shape
        dev = self.codes.device
        qweight = torch.empty((n, (d * self.bits + 31) // 32), dtype=torch.int32, device=dev)
        s16 = torch.empty(self.scales.shape, dtype=torch.int16, device=dev)
        z16 = torch.empty(self.zeros.shape, dtype=torch.int16, device=dev)
        L.gptq_pack(self.codes, self.bits, self.scales, self.zeros, qweight, s16, z16)
        return qweight, s16.view(torch.float16), z16.view(torch.float16)


def hessian(X: torch.Tensor, H: torch.Tensor | None = None, accumulate: bool = False,
            dev_status: torch.Tensor | None = None) -> torch.Tensor:
    """H (upper triangle) = 2 X^T X for token-major X [n_tokens, d_in] (bf16 or fp32)."""
    d = X.shape[1]
    if H is None:
        H = torch.empty((d, d), dtype=torch.float32, device=X.device)
    L.gptq_hessian_accumulate(H, X, 2.0, accumulate, dev_status)
    return H


def check_status(dev_status: torch.Tensor) -> None:
    code, index = (int(v) for v in dev_status.cpu().tolist())
    if code != 0:
        raise L.GPTQError(code, f"device (index {index})")


def quantize_layer(W: torch.Tensor, X: torch.Tensor | None = None, H: torch.Tensor | None = None,
                   bits: int = 4, group_size: int = 128, sym: bool = False,
                   act_order: bool = False, perm: torch.Tensor | None = None,
                   percdamp: float = 0.01, prepared: tuple | None = None,
                   check: bool = True, static_groups: bool = False) -> QuantizedLayer:
    """GPTQ of one linear layer. Give X (calibration activations), or H (raw 2 X^T X, clobbered),
    or prepared = (U, perm, dead) from prepare() to share one Hessian between layers.
    static_groups: groups in original column order with parameters from the original weights."""
    n, d = W.shape
    dev = W.device
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    order = L.GPTQ_ORDER_GIVEN if perm is not None else (
        L.GPTQ_ORDER_DESC_ACT if act_order else L.GPTQ_ORDER_NATURAL)
    p = L.make_params(bits, group_size, sym, order, 128, percdamp, static_groups)
    ws = torch.empty(L.gptq_workspace_size(n, d, p), dtype=torch.uint8, device=dev)
    if prepared is None:
        if H is None:
            H = hessian(X, dev_status=status)
        U, perm, dead = prepare(H, p, perm=perm, ws=ws, dev_status=status)
    else:
        U, perm, dead = prepared
    G = 1 if group_size == -1 else d // group_size
    codes = torch.empty((n, d), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, G), dtype=torch.float32, device=dev)
    zeros = torch.empty((n, G), dtype=torch.float32, device=dev)
    g_idx = torch.empty(d, dtype=torch.int32, device=dev)
    L.gptq_quantize_layer(W, U, perm, dead, p, codes, scales, zeros, g_idx, ws, status)
    if check:
        check_status(status)
    return QuantizedLayer(codes, scales, zeros, g_idx, perm, dead, bits, group_size)


def prepare(H: torch.Tensor, params, perm: torch.Tensor | None = None, ws=None, dev_status=None):
    """(U, perm, dead) from a raw Hessian (H is clobbered)."""
    d = H.shape[0]
    dev = H.device
    U = torch.empty((d, d), dtype=torch.float32, device=dev)
    if perm is None:
        perm = torch.empty(d, dtype=torch.int32, device=dev)
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    L.gptq_prepare_hinv(H, params, U, perm, dead, ws, dev_status)
    return U, perm, dead


def rtn(W: torch.Tensor, bits: int = 4, group_size: int = 128, sym: bool = False):
    n, d = W.shape
    G = 1 if group_size == -1 else d // group_size
    codes = torch.empty((n, d), dtype=torch.uint8, device=W.device)
    scales = torch.empty((n, G), dtype=torch.float32, device=W.device)
    zeros = torch.empty((n, G), dtype=torch.float32, device=W.device)
    L.rtn_quantize(W, L.make_params(bits, group_size, sym), codes, scales, zeros)
    return codes, scales, zeros
