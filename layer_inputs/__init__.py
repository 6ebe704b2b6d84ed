"""Seeded synthetic inputs for GPTQ layer quantization: weights W and calibration activations X.

This module only draws random numbers and lays them out; it contains none of the
quantization arithmetic. Both the FP64 oracle (tests) and the CUDA path (tests, bench)
consume exactly the bytes produced here.

Layouts
  W : [d_out, d_in] row-major, bf16 (stored as torch.bfloat16) or fp32.
  X : token-major [N, d_in] row-major (one row per calibration token). The pages write the
      calibration matrix as X in R^{d_in x N}; the token-major array is the same memory read
      column-major, and H = 2 X X^T becomes 2 * X_tm^T X_tm.

Distributions (per workload table below)
  W_ij ~ N(0, sigma_w^2), rounded once to the storage dtype (RNE).
  X_ti = z_ti * c_i with z ~ N(0,1) (or |N(0,1)| for ReLU-like inputs), channel scale
  c_i ~ LogNormal(0, sigma_c); a seeded random subset of round(frac*d) channels (the first
  entries of a seeded permutation) is multiplied by an outlier factor.

Every stream is a numpy PCG64 seeded from SeedSequence(entropy=seed, spawn_key=(chunk,)), so
the bytes do not depend on the number of threads used to draw them.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np
import torch

_CHUNK_ROWS = 4096


def _rng(seed: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(entropy=seed, spawn_key=(chunk,))))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def channel_scales(d: int, chan_sigma: float, outlier_frac: float, outlier_mult: float,
                   seed: int) -> np.ndarray:
    """Per-channel scale c_i (float32): lognormal(0, chan_sigma) with outlier channels."""
    rng = _rng(seed, 1 << 30)
    c = rng.lognormal(0.0, chan_sigma, size=d).astype(np.float64)
    n_out = int(round(outlier_frac * d))
    if n_out > 0:
        idx = rng.permutation(d)[:n_out]
        c[idx] *= outlier_mult
    return c.astype(np.float32)


def outlier_channels(d: int, chan_sigma: float, outlier_frac: float, seed: int) -> np.ndarray:
    """Indices of the outlier channels chosen by channel_scales (same stream, same order)."""
    rng = _rng(seed, 1 << 30)
    rng.lognormal(0.0, chan_sigma, size=d)
    n_out = int(round(outlier_frac * d))
    return np.sort(rng.permutation(d)[:n_out]) if n_out > 0 else np.zeros(0, np.int64)


def _to_dtype(a: np.ndarray, dtype: torch.dtype, out: torch.Tensor | None, row0: int) -> torch.Tensor:
    t = torch.from_numpy(a)
    if out is not None:
        out[row0:row0 + a.shape[0]].copy_(t)  # RNE conversion when out is bf16
        return out
    return t.to(dtype)


def weight(d_out: int, d_in: int, sigma: float, dtype: torch.dtype, seed: int) -> torch.Tensor:
    """W ~ N(0, sigma^2), [d_out, d_in], rounded once to `dtype` (CPU tensor)."""
    out = torch.empty((d_out, d_in), dtype=dtype)

    def fill(chunk: int) -> None:
        r0 = chunk * _CHUNK_ROWS
        r1 = min(d_out, r0 + _CHUNK_ROWS)
        a = _rng(seed, chunk).standard_normal((r1 - r0, d_in), dtype=np.float32)
        a *= np.float32(sigma)
        out[r0:r1].copy_(torch.from_numpy(a))

    n_chunks = (d_out + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(n_chunks)))
    return out


def activations(n_tokens: int, d: int, *, chan_sigma: float, outlier_frac: float = 0.0,
                outlier_mult: float = 1.0, half_normal: bool = False,
                dtype: torch.dtype = torch.bfloat16, seed: int,
                out: torch.Tensor | None = None) -> torch.Tensor:
    """Token-major calibration activations X [n_tokens, d] (CPU tensor, optionally into `out`,
    e.g. a pinned buffer)."""
    c = channel_scales(d, chan_sigma, outlier_frac, outlier_mult, seed)
    if out is None:
        out = torch.empty((n_tokens, d), dtype=dtype)
    assert out.shape == (n_tokens, d) and out.dtype == dtype

    def fill(chunk: int) -> None:
        r0 = chunk * _CHUNK_ROWS
        r1 = min(n_tokens, r0 + _CHUNK_ROWS)
        a = _rng(seed, chunk).standard_normal((r1 - r0, d), dtype=np.float32)
        if half_normal:
            np.abs(a, out=a)
        a *= c[None, :]
        out[r0:r1].copy_(torch.from_numpy(a))

    n_chunks = (n_tokens + _CHUNK_ROWS - 1) // _CHUNK_ROWS
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill, range(n_chunks)))
    return out


# ----------------------------------------------------------------------------------------------
# Workload table: the five layer shapes of the benchmark, each with its synthetic inputs.
# ----------------------------------------------------------------------------------------------

@dataclass(frozen=True)
class ActSpec:
    """One calibration input X [n_tokens, d]."""
    name: str
    d: int
    n_tokens: int
    chan_sigma: float
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    half_normal: bool = False
    dtype: str = "bf16"
    seed: int = 0

    def make(self, out: torch.Tensor | None = None) -> torch.Tensor:
        return activations(self.n_tokens, self.d, chan_sigma=self.chan_sigma,
                           outlier_frac=self.outlier_frac, outlier_mult=self.outlier_mult,
                           half_normal=self.half_normal, dtype=_dtype(self.dtype), seed=self.seed,
                           out=out)


@dataclass(frozen=True)
class LinearSpec:
    """One linear layer W [d_out, d_in] quantized against the Hessian of input `act`."""
    name: str
    d_out: int
    d_in: int
    sigma: float
    act: str
    dtype: str = "bf16"
    seed: int = 0

    def make(self) -> torch.Tensor:
        return weight(self.d_out, self.d_in, self.sigma, _dtype(self.dtype), self.seed)


@dataclass(frozen=True)
class QuantSpec:
    bits: int = 4
    group_size: int = 128      # -1: one scale per output row
    sym: bool = False
    act_order: bool = False
    block_size: int = 128
    percdamp: float = 0.01


@dataclass(frozen=True)
class Workload:
    name: str
    acts: tuple[ActSpec, ...]
    linears: tuple[LinearSpec, ...]
    quant: QuantSpec = field(default_factory=QuantSpec)

    def act(self, name: str) -> ActSpec:
        return next(a for a in self.acts if a.name == name)

    @property
    def n_weights(self) -> int:
        return sum(l.d_out * l.d_in for l in self.linears)


def _dtype(s: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[s]


def _workloads() -> dict[str, Workload]:
    w = {}
    # 1: one small fp32 layer, 2048 tokens, lognormal(0, 0.5) channel scales.
    w["tiny_256"] = Workload(
        "tiny_256",
        acts=(ActSpec("x", 256, 2048, 0.5, dtype="f32", seed=1001),),
        linears=(LinearSpec("w", 256, 256, 0.02, "x", dtype="f32", seed=1002),),
        quant=QuantSpec(bits=4, group_size=128))
    # 2: Llama-7B attention projection, 128 x 2048 calibration tokens, 0.1 % outlier channels x20.
    w["llama7b_attn_proj"] = Workload(
        "llama7b_attn_proj",
        acts=(ActSpec("x", 4096, 262144, 1.0, 0.001, 20.0, seed=2001),),
        linears=(LinearSpec("w", 4096, 4096, 0.02, "x", seed=2002),),
        quant=QuantSpec(bits=4, group_size=128))
    # 3: Llama-7B MLP: gate/up share the attention-shaped input; down sees a ReLU-like input.
    w["llama7b_mlp"] = Workload(
        "llama7b_mlp",
        acts=(ActSpec("x_gu", 4096, 262144, 1.0, 0.001, 20.0, seed=3001),
              ActSpec("x_down", 11008, 262144, 1.0, 0.001, 20.0, half_normal=True, seed=3002)),
        linears=(LinearSpec("gate", 11008, 4096, 0.02, "x_gu", seed=3003),
                 LinearSpec("up", 11008, 4096, 0.02, "x_gu", seed=3004),
                 LinearSpec("down", 4096, 11008, 0.02, "x_down", seed=3005)),
        quant=QuantSpec(bits=3, group_size=128, act_order=True))
    # 4: Llama-13B decoder block, 7 linears, four distinct inputs of 131072 tokens.
    w["llama13b_block"] = Workload(
        "llama13b_block",
        acts=(ActSpec("x_qkv", 5120, 131072, 1.0, 0.001, 20.0, seed=4001),
              ActSpec("x_o", 5120, 131072, 1.0, 0.001, 20.0, seed=4002),
              ActSpec("x_gu", 5120, 131072, 1.0, 0.001, 20.0, seed=4003),
              ActSpec("x_down", 13824, 131072, 1.0, 0.001, 20.0, seed=4004)),
        linears=(LinearSpec("q", 5120, 5120, 0.02, "x_qkv", seed=4011),
                 LinearSpec("k", 5120, 5120, 0.02, "x_qkv", seed=4012),
                 LinearSpec("v", 5120, 5120, 0.02, "x_qkv", seed=4013),
                 LinearSpec("o", 5120, 5120, 0.02, "x_o", seed=4014),
                 LinearSpec("gate", 13824, 5120, 0.02, "x_gu", seed=4015),
                 LinearSpec("up", 13824, 5120, 0.02, "x_gu", seed=4016),
                 LinearSpec("down", 5120, 13824, 0.02, "x_down", seed=4017)),
        quant=QuantSpec(bits=4, group_size=128))
    # 5: Llama-70B down projection, ReLU-like input with 0.05 % outlier channels x30,
    # 4-bit symmetric with one scale per output row.
    w["llama70b_down_proj"] = Workload(
        "llama70b_down_proj",
        acts=(ActSpec("x", 28672, 131072, 1.0, 0.0005, 30.0, half_normal=True, seed=5001),),
        linears=(LinearSpec("w", 8192, 28672, 0.015, "x", seed=5002),),
        quant=QuantSpec(bits=4, group_size=-1, sym=True))
    return w


WORKLOADS: dict[str, Workload] = _workloads()
