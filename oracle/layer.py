"""One linear layer end to end — oracle.

Follows the order of [GPTQ-MATH] §GPTQ Algorithm Execution Walkthrough with the act-order
workflow of §Activation Ordering around it: (permute) -> dead-column fix -> damping -> U ->
sweep -> codes returned in the original column order with g_idx (the group of each original
column: g_idx[pi[k]] = k // g).
"""
from __future__ import annotations

import numpy as np

from . import prepare as prep
from . import quantizer as qz
from . import sweep as sw


def gptq_layer(W: np.ndarray, H: np.ndarray, bits: int = 4, group_size: int = 128,
               sym: bool = False, act_order: bool = False, block_size: int = 128,
               percdamp: float = 0.01, perm: np.ndarray | None = None, route: str = "blocked"):
    """GPTQ of one layer in float64. Returns dict(codes uint8 [n,d] original order, S, Z
    [n, G] in sweep-group order, g_idx int [d], perm, dead (sweep order), U, lam, Err)."""
    P = prep.prepare(H, W, percdamp=percdamp, act_order=act_order, perm=perm)
    Wp, U = P["W"], P["U"]
    if route == "blocked":
        c, S, Z, Err = sw.sweep_blocked(Wp, U, bits, group_size, sym, block_size)
    elif route == "chol":
        c, S, Z, Err = sw.sweep_chol(Wp, U, bits, group_size, sym)
    elif route == "obs":
        c, S, Z, _ = sw.sweep_obs(Wp, P["H_inv"], bits, group_size, sym)
        Err = None
    else:
        raise ValueError(route)
    d = Wp.shape[1]
    perm = P["perm"]
    codes = np.empty_like(c)
    codes[:, perm] = c
    g = d if group_size == -1 else group_size
    g_idx = np.empty(d, np.int64)
    g_idx[perm] = np.arange(d) // g if group_size != -1 else 0
    return dict(codes=codes, S=S, Z=Z, g_idx=g_idx, perm=perm, dead=P["dead"], U=U,
                lam=P["lam"], Err=Err)


def rtn_layer(W: np.ndarray, bits: int = 4, group_size: int = 128, sym: bool = False):
    """RTN of one layer in W's dtype (float32 for bit-exact parity); natural group order."""
    codes, S, Z = qz.rtn(W, bits, group_size, sym)
    d = W.shape[1]
    g_idx = np.zeros(d, np.int64) if group_size == -1 else np.arange(d) // group_size
    return dict(codes=codes, S=S, Z=Z, g_idx=g_idx)
