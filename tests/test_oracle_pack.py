"""Pins for oracle/pack.py (no GPU)."""
import struct

import numpy as np
import pytest

from conftest import parse_vector, read_golden
from oracle import pack as pk


def test_hand_words():
    g = read_golden("pack_hand.txt")
    c4 = np.array([parse_vector(g["bits4_codes"], int)], np.uint8)
    assert pk.pack_rows(c4, 4)[0].tolist() == [int(g["bits4_words"], 16)]
    c3 = np.array([parse_vector(g["bits3_codes"], int)], np.uint8)
    w3 = pk.pack_rows(c3, 3)
    assert w3.shape == (1, 3)
    assert int(w3[0, 0]) == int(g["bits3_word0"], 16)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("d", [32, 128, 200, 4096])
def test_round_trip(bits, d):
    rng = np.random.default_rng(bits * 1000 + d)
    codes = rng.integers(0, 2 ** bits, (5, d), dtype=np.uint8)
    w = pk.pack_rows(codes, bits)
    assert w.shape == (5, (d * bits + 31) // 32)
    np.testing.assert_array_equal(pk.unpack_rows(w, d, bits), codes)


def test_bit_rate_4_25():
    """[GPTQ-MATH] §Quantization Formats and Group Size: b + 32/g = 4.25 bits/weight at b=4, g=128."""
    assert pk.bits_per_weight(4096, 4096, 4, 4096 // 128) == 4.25
    assert pk.bits_per_weight(11008, 4096, 3, 32) == 3.25


def test_fp16_against_python_half_encoder():
    """float32 -> fp16 bits agree with struct 'e' (CPython's own IEEE binary16 encoder) on
    normals, subnormals, overflow and exact ties."""
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.normal(0, 1e-3, 20000), rng.lognormal(0, 4, 20000) * rng.choice([-1, 1], 20000),
        np.array([0.0, -0.0, 65504.0, 65519.0, 65520.0, 6.0e-8, 2.0 ** -24 * 1.5, 2.0 ** -25,
                  1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 8.0, 15.0, 1e9])]).astype(np.float32)
    got = pk.to_fp16_bits(vals)
    for v, b in zip(vals.tolist(), got.tolist()):
        try:
            ref = struct.unpack("<H", struct.pack("<e", v))[0]
        except OverflowError:
            ref = 0x7C00 if v > 0 else 0xFC00
        assert b == ref, (v, hex(b), hex(ref))
