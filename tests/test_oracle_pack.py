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


def _half_rne_binade(sign: int, e: int, mant: np.ndarray) -> np.ndarray:
    """IEEE binary32 -> binary16 bit patterns, round to nearest even, written from the format
    definitions for the fp32 patterns (sign, biased exponent e, significand bits mant) of one
    normal binade: the value is m * 2^(e - 150) with m = 2^23 + mant. It is rounded to a
    multiple of the binary16 quantum of that binade (2^(p - 10) for a normal result in binade
    2^p, 2^-24 for a subnormal one), ties to even; a result of 2^16 - 2^4 = 65520 or more is
    infinity."""
    p = e - 127
    quantum_exp = max(p, -14) - 10
    shift = quantum_exp - (e - 150)                 # significand bits below the quantum, >= 13
    u = np.uint32
    m = mant | u(1 << 23)                           # 24-bit significand
    q = m >> u(shift)
    rem = m & u((1 << shift) - 1)
    half = u(1 << (shift - 1))
    q += ((rem > half) | ((rem == half) & ((q & u(1)) == 1))).astype(np.uint32)
    if quantum_exp == -24:                          # subnormal binade: q quanta of 2^-24
        bits = q                                    # q == 1024 encodes the smallest normal
    else:                                           # q in [1024, 2048]: 2048 carries into E + 1
        bits = (u(p + 15) << u(10)) + (q - u(1024))
    np.minimum(bits, u(0x7C00), out=bits)           # overflow to infinity
    return (bits | u(sign << 15)).astype(np.uint16)


def test_fp16_rne_brute_force_over_the_half_range():
    """Every fp32 pattern of both signs in the binades 2^-26 .. 2^15 (where binary16 results
    are finite and nonzero, or the ties and roundings at the edges: 42 binades x 2^23
    significands x 2 signs), converted by the oracle, equals the conversion written from the
    IEEE definitions."""
    step = 1 << 20
    for c0 in range(0, 1 << 23, step):
        mant = np.arange(c0, c0 + step, dtype=np.uint32)
        for sign in (0, 1):
            for e in range(127 - 26, 127 + 16):
                pat = np.uint32(sign << 31) | np.uint32(e << 23) | mant
                got = pk.to_fp16_bits(pat.view(np.float32))
                ref = _half_rne_binade(sign, e, mant)
                bad = np.nonzero(got != ref)[0]
                assert bad.size == 0, (sign, e, hex(int(pat[bad[0]])), hex(int(got[bad[0]])),
                                       hex(int(ref[bad[0]])))
    # Outside that range: below 2^-26 everything rounds to a signed zero; from 2^16 up, infinity.
    tiny = np.array([2.0 ** -27, 1e-30, 1e-45, -2.0 ** -27], np.float32)
    assert pk.to_fp16_bits(tiny).tolist() == [0, 0, 0, 0x8000]
    big = np.array([65536.0, 1e30, -65536.0], np.float32)
    assert pk.to_fp16_bits(big).tolist() == [0x7C00, 0x7C00, 0xFC00]
