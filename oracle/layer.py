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
               percdamp: float = 0.01, perm: np.ndarray | None = None, route: str = "blocked",
               static_groups: bool = False):
    """GPTQ of one layer in float64. Returns dict(codes uint8 [n,d] original order, S, Z
    [n, G], g_idx int [d], perm, dead (sweep order), U, lam, Err). S and Z are in sweep-group
    order (g_idx[pi[k]] = k // g), or with static_groups in original group order
    (g_idx[c] = c // g), computed from the dead-column-fixed weights before the sweep."""
    P = prep.prepare(H, W, percdamp=percdamp, act_order=act_order, perm=perm)
    Wp, U = P["W"], P["U"]
    d = Wp.shape[1]
    perm = P["perm"]
    static = None
    if static_groups:
        if group_size == -1:
            raise ValueError("static groups need a group size")
        W_orig = np.empty_like(Wp)
        W_orig[:, perm] = Wp                      # dead-fixed weights in the original order
        S0, Z0 = sw.static_group_params(W_orig, bits, group_size, sym)
        static = (S0, Z0, np.asarray(perm) // group_size)
    if route == "blocked":
        c, S, Z, Err = sw.sweep_blocked(Wp, U, bits, group_size, sym, block_size, static=static)
    elif route == "chol":
        c, S, Z, Err = sw.sweep_chol(Wp, U, bits, group_size, sym, static=static)
    elif route == "obs":
        c, S, Z, _ = sw.sweep_obs(Wp, P["H_inv"], bits, group_size, sym, static=static)
        Err = None
    else:
        raise ValueError(route)
    codes = np.empty_like(c)
    codes[:, perm] = c
    g = d if group_size == -1 else group_size
    g_idx = np.empty(d, np.int64)
    if static_groups:
        g_idx[:] = np.arange(d) // g
    else:
        g_idx[perm] = np.arange(d) // g if group_size != -1 else 0
    return dict(codes=codes, S=S, Z=Z, g_idx=g_idx, perm=perm, dead=P["dead"], U=U,
                lam=P["lam"], Err=Err)


def rtn_layer(W: np.ndarray, bits: int = 4, group_size: int = 128, sym: bool = False):
    """RTN of one layer in W's dtype (float32 for bit-exact parity); natural group order."""
    codes, S, Z = qz.rtn(W, bits, group_size, sym)
    d = W.shape[1]
    g_idx = np.zeros(d, np.int64) if group_size == -1 else np.arange(d) // group_size
    return dict(codes=codes, S=S, Z=Z, g_idx=g_idx)
