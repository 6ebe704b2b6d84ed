"""Data-parallel GPTQ of one layer over a torch.distributed group, one process per GPU.

The method shards with a single exchange:

* Tokens. H = 2 X^T X is a sum over calibration tokens ("GPTQ: Mathematical Foundations ...",
  §Second-Order Taylor Expansion; "INT4 and GPTQ Quantization", §The Quantization Error and
  Layerwise Objective), so each rank forms the upper triangle of its own tokens' sum with
  gptq_hessian_accumulate and one all-reduce (sum) over the group gives every rank the whole H.
* Prepare. Replicated: every rank runs gptq_prepare_hinv on the same bits of H, and the
  kernels are deterministic, so every rank holds the same U, permutation and dead columns.
* Rows. Given U, the column sweep treats the rows of W independently (each row's error only
  updates that row; "GPTQ: Mathematical Foundations ...", §2 Lazy Batch Updates), so each rank
  quantizes and packs a contiguous slice of rows, with no exchange.
* Gather (optional). One all-gather of the packed words and fp16 parameters puts the whole
  packed layer on every rank.

The shard plan, the all-reduce and the gather are plain host logic over torch.distributed and
work on tensors of any device; the arithmetic is the library's (quantize_layer_sharded).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import _lib as L
from .layer import QuantizedLayer, check_status


def split_range(total: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """[start, stop) of rank's share of `total` items: contiguous, in rank order, covering
    [0, total) exactly once. Shares are balanced in whole units of `align` items (unit counts
    differ by at most one); the share that reaches `total` is cut there."""
    if world < 1 or not 0 <= rank < world or align < 1 or total < 0:
        raise ValueError("bad split")
    units = -(-total // align)                 # ceil(total / align)
    base, extra = divmod(units, world)
    start = align * (rank * base + min(rank, extra))
    stop = align * ((rank + 1) * base + min(rank + 1, extra))
    return min(start, total), min(stop, total)


@dataclass(frozen=True)
class ShardPlan:
    """Which calibration tokens and which rows of W a rank owns."""
    world: int
    rank: int
    n_tokens: int
    n_rows: int
    tokens: tuple[int, int]
    rows: tuple[int, int]

    def rows_of(self, rank: int) -> tuple[int, int]:
        return split_range(self.n_rows, self.world, rank, 16)

    @property
    def max_rows(self) -> int:
        return max(b - a for a, b in map(self.rows_of, range(self.world)))


def plan(n_tokens: int, n_rows: int, world: int, rank: int) -> ShardPlan:
    """Token shares are multiples of 16 tokens (one SYRK k-step); row shares multiples of 16
    rows (one sweep CTA). Every rank must own rows (n_rows > 16 * (world - 1)); a rank may own
    no tokens."""
    if n_rows <= 16 * (world - 1):
        raise ValueError(f"{n_rows} rows leave a rank of {world} without rows")
    return ShardPlan(world, rank, n_tokens, n_rows, split_range(n_tokens, world, rank, 16),
                     split_range(n_rows, world, rank, 16))


def allreduce_hessian(H: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partial H in place. Only the upper triangle carries data; the caller
    allocates H zeroed, so the strictly lower triangle (never written by the library) adds up to
    zero. The whole square is reduced: d^2 fp32 values per rank."""
    if not H.is_contiguous():
        raise ValueError("H must be contiguous")
    dist.all_reduce(H, op=dist.ReduceOp.SUM, group=group)
    return H


def gather_rows(local: torch.Tensor, p: ShardPlan, group=None) -> torch.Tensor:
    """Concatenate every rank's row slice (rank order) on every rank. `local` holds this rank's
    p.rows[1] - p.rows[0] rows; slices are padded to the largest share for the all-gather."""
    r0, r1 = p.rows
    if local.shape[0] != r1 - r0:
        raise ValueError("local rows do not match the plan")
    m = p.max_rows
    padded = torch.zeros((m,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    padded[: r1 - r0] = local
    out = torch.empty((p.world * m,) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    dist.all_gather_into_tensor(out, padded, group=group)
    parts = []
    for r in range(p.world):
        a, b = p.rows_of(r)
        parts.append(out[r * m: r * m + (b - a)])
    return torch.cat(parts, 0)


def quantize_layer_sharded(W_rows: torch.Tensor, X_tokens: torch.Tensor, p: ShardPlan,
                           bits: int = 4, group_size: int = 128, sym: bool = False,
                           act_order: bool = False, percdamp: float = 0.01,
                           static_groups: bool = False, gather: bool = False, group=None):
    """GPTQ of one layer sharded over `group` on this rank's GPU.

    W_rows: this rank's rows of W (p.rows), bf16 or fp32 on the device. X_tokens: this rank's
    calibration tokens (p.tokens), token-major [tokens, d_in]. Returns the QuantizedLayer of this
    rank's rows and, with gather=True, the whole packed layer (qweight, scales fp16, zeros fp16)
    on every rank. Every rank must make the same call (the collectives are matched)."""
    d = X_tokens.shape[1]
    if W_rows.shape[1] != d or W_rows.shape[0] != p.rows[1] - p.rows[0]:
        raise ValueError("W_rows does not match the plan")
    if X_tokens.shape[0] != p.tokens[1] - p.tokens[0]:
        raise ValueError("X_tokens does not match the plan")
    dev = X_tokens.device
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    H = torch.zeros((d, d), dtype=torch.float32, device=dev)
    if X_tokens.shape[0] > 0:
        L.gptq_hessian_accumulate(H, X_tokens, 2.0, False, status)
    allreduce_hessian(H, group)
    order = L.GPTQ_ORDER_DESC_ACT if act_order else L.GPTQ_ORDER_NATURAL
    prm = L.make_params(bits, group_size, sym, order, 128, percdamp, static_groups)
    n = W_rows.shape[0]
    ws = torch.empty(L.gptq_workspace_size(n, d, prm), dtype=torch.uint8, device=dev)
    U = torch.empty((d, d), dtype=torch.float32, device=dev)
    perm = torch.empty(d, dtype=torch.int32, device=dev)
    dead = torch.empty(d, dtype=torch.uint8, device=dev)
    L.gptq_prepare_hinv(H, prm, U, perm, dead, ws, status)
    G = 1 if group_size == -1 else d // group_size
    codes = torch.empty((n, d), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, G), dtype=torch.float32, device=dev)
    zeros = torch.empty((n, G), dtype=torch.float32, device=dev)
    g_idx = torch.empty(d, dtype=torch.int32, device=dev)
    L.gptq_quantize_layer(W_rows, U, perm, dead, prm, codes, scales, zeros, g_idx, ws, status)
    check_status(status)
    out = QuantizedLayer(codes, scales, zeros, g_idx, perm, dead, bits, group_size)
    if not gather:
        return out
    qweight, s16, z16 = out.pack()
    return out, (gather_rows(qweight, p, group), gather_rows(s16, p, group),
                 gather_rows(z16, p, group))
