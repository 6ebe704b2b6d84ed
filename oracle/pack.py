"""Storage format: packed codes and fp16 metadata — oracle.

[GPTQ-MATH] §Inference Execution and Modern Kernel Architectures: eight 4-bit weights are packed
into one int32 word. [INT4-GPTQ] §Group Quantization: scale and zero kept in FP16 for
dequantization. [GPTQ-MATH] §Quantization Formats and Group Size: b + (16 + 16)/g bits per weight.

Reading (the pages fix only the 4-bit case): each output row is one LSB-first bit stream along
d_in; code k occupies bits [b*k, b*k + b) of the stream, and word w holds stream bits
[32w, 32w + 32) with stream bit 32w + t at bit t. For b = 4 this is code k at bits 4(k mod 8) of
word k/8; for b = 3 it is 32 codes per 3 words. A row's tail word is zero-padded.

Pinned by: hand-packed words (tests/golden/pack_hand.txt), pack/unpack round trip, the 4.25
bits/weight figure for b = 4, g = 128, and fp16 conversion against Python's own IEEE half
encoder (struct format 'e').
"""
from __future__ import annotations

import numpy as np


def words_per_row(d: int, bits: int) -> int:
    return (d * bits + 31) // 32


def pack_rows(codes: np.ndarray, bits: int) -> np.ndarray:
    """codes uint8 [n, d] (each < 2^bits) -> uint32 [n, ceil(d*bits/32)]."""
    codes = np.asarray(codes, np.uint8)
    n, d = codes.shape
    nw = words_per_row(d, bits)
    stream = ((codes[:, :, None] >> np.arange(bits, dtype=np.uint8)) & 1).reshape(n, d * bits)
    padded = np.zeros((n, nw * 32), np.uint64)
    padded[:, :d * bits] = stream
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (padded.reshape(n, nw, 32) * weights).sum(axis=2).astype(np.uint32)


def unpack_rows(words: np.ndarray, d: int, bits: int) -> np.ndarray:
    """Inverse of pack_rows."""
    words = np.asarray(words, np.uint32)
    n, nw = words.shape
    stream = ((words[:, :, None].astype(np.uint64) >> np.arange(32, dtype=np.uint64)) & 1)
    stream = stream.reshape(n, nw * 32)[:, :d * bits].reshape(n, d, bits)
    return (stream * (np.uint64(1) << np.arange(bits, dtype=np.uint64))).sum(axis=2).astype(np.uint8)


def to_fp16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> IEEE binary16 bit patterns (round to nearest even), as uint16."""
    with np.errstate(over="ignore"):
        return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def pack(codes: np.ndarray, scales: np.ndarray, zeros: np.ndarray, bits: int):
    """(qweight uint32 [n, words], scales fp16 bits [n, G], zeros fp16 bits [n, G])."""
    return pack_rows(codes, bits), to_fp16_bits(scales), to_fp16_bits(zeros)


def bits_per_weight(d_out: int, d_in: int, bits: int, n_groups: int) -> float:
    """Storage bits per weight of the packed layer: code words plus 16-bit scale and zero."""
    total = d_out * words_per_row(d_in, bits) * 32 + d_out * n_groups * (16 + 16)
    return total / (d_out * d_in)
