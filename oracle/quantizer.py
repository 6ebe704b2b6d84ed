"""Uniform quantizer, group statistics and round-to-nearest (RTN) — oracle.

[INT4-GPTQ] §Uniform INT4 Quantization: w_hat = s (q - z), s = (max - min)/(2^b - 1);
  symmetric: s = max|W| / (2^(b-1) - 1), q = clamp(round(w/s), -2^(b-1), 2^(b-1) - 1).
[INT4-GPTQ] §Group Quantization: one (s, z) per run of g consecutive weights of a row;
  z = clamp(round(-min/s), 0, 2^b - 1); codes stored unsigned, s and z kept for dequantization.
[GPTQ-MATH] §Quantization Formats and Group Size: q = clamp(round(w/s) + z, 0, 2^b - 1),
  symmetric z = 0 (or 2^(b-1)); per-channel (one scale per output row) vs group-wise.
[Q-INT8] §Deriving the scale and zero-point: s = (x_max - x_min)/(q_max - q_min),
  z = round(q_min - x_min/s).

Readings of the pages used here:
  * q = clamp(rne(w/s) + z) (round first, then add the integer zero-point), as two of the
    three pages write it; round-half-to-even for every rounding.
  * A degenerate range (s == 0: max == min, or max|w| == 0) uses s = 1.
  * Symmetric codes are stored unsigned as q + 2^(b-1) with zero-point z = 2^(b-1), so one
    dequantization formula s (code - z) serves both modes.
  * The arithmetic runs in the dtype of the inputs: float32 for RTN / quantize-given-scales
    (the pages' tensor code is float32), float64 inside the oracle sweep.

Pinned by: the worked INT8 example of [Q-INT8] (tests/golden/int8_worked_example.txt), hand
cases for 4-bit asymmetric groups, endpoint and half-step error properties.
"""
from __future__ import annotations

import numpy as np


def maxq(bits: int) -> int:
    return (1 << bits) - 1


def asym_params(wmin: np.ndarray, wmax: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """(s, z) of the asymmetric min/max quantizer, computed in the dtype of wmin/wmax."""
    dt = np.result_type(wmin, wmax)
    wmin = np.asarray(wmin, dt)
    wmax = np.asarray(wmax, dt)
    s = (wmax - wmin) / dt.type(maxq(bits))
    s = np.where(s == 0, dt.type(1), s).astype(dt)
    z = np.clip(np.rint(-wmin / s), dt.type(0), dt.type(maxq(bits))).astype(dt)
    return s, z


def sym_params(amax: np.ndarray, bits: int) -> tuple[np.ndarray, np.ndarray]:
    """(s, z) of the symmetric quantizer; z = 2^(b-1) is the unsigned storage offset."""
    dt = np.asarray(amax).dtype
    amax = np.asarray(amax, dt)
    s = amax / dt.type((1 << (bits - 1)) - 1)
    s = np.where(s == 0, dt.type(1), s).astype(dt)
    z = np.full_like(s, dt.type(1 << (bits - 1)))
    return s, z


def quantize(w: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """Unsigned code q = clamp(rne(w/s) + z, 0, 2^b - 1), in the dtype of w (returned as float)."""
    dt = w.dtype
    return np.clip(np.rint(w / s) + z, dt.type(0), dt.type(maxq(bits)))


def dequantize(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """w_hat = s (q - z)."""
    return s * (q - z)


def params_from_values(vals: np.ndarray, bits: int, sym: bool) -> tuple[np.ndarray, np.ndarray]:
    """(s, z) for each row of `vals` (statistics over the last axis)."""
    if sym:
        return sym_params(np.max(np.abs(vals), axis=-1), bits)
    return asym_params(np.min(vals, axis=-1), np.max(vals, axis=-1), bits)


def rtn(W: np.ndarray, bits: int, group_size: int, sym: bool):
    """Round-to-nearest baseline: statistics from the original W, then quantize every weight.

    [GPTQ-MATH] §Comparison: RTN rounds each weight independently; group statistics as in
    [INT4-GPTQ] §Group Quantization. group_size == -1 gives one scale per output row.
    Runs in W's dtype (float32 for bit-exact parity).
    Returns codes uint8 [n, d], scales [n, G], zeros [n, G].
    """
    n, d = W.shape
    g = d if group_size == -1 else group_size
    G = (d + g - 1) // g
    codes = np.empty((n, d), np.uint8)
    S = np.empty((n, G), W.dtype)
    Z = np.empty((n, G), W.dtype)
    for gi in range(G):
        c0, c1 = gi * g, min(d, gi * g + g)
        s, z = params_from_values(W[:, c0:c1], bits, sym)
        S[:, gi] = s
        Z[:, gi] = z
        codes[:, c0:c1] = quantize(W[:, c0:c1], s[:, None], z[:, None], bits).astype(np.uint8)
    return codes, S, Z
