"""Pins for oracle/quantizer.py against what the pages fix (no GPU)."""
import numpy as np
import pytest

from conftest import parse_vector, read_golden
from oracle import quantizer as qz


def test_int8_worked_example():
    """[Q-INT8] Worked example 1: [-0.9, 0.1, 0.6] -> s = 0.9/127, q = [-127, 14, 85]."""
    g = read_golden("int8_worked_example.txt")
    bits = int(g["bits"])
    w = np.array(parse_vector(g["w"]), np.float32)
    s, z = qz.sym_params(np.max(np.abs(w)), bits)
    assert s.dtype == np.float32
    assert abs(float(s) - float(g["s"])) < 5e-6
    code = qz.quantize(w, s, z, bits)
    q_signed = code - z
    assert q_signed.tolist() == parse_vector(g["q_signed"])
    w_hat = qz.dequantize(code, s, z)
    np.testing.assert_allclose(w_hat, parse_vector(g["w_hat"]), atol=4e-4)
    np.testing.assert_allclose(np.abs(w - w_hat), parse_vector(g["abs_err"]), atol=4e-4)


def test_asym_hand_case_4bit():
    """Group spanning [-0.75, 0.75] at 4 bits: s = 1.5/15 = 0.1, z = rne(7.5) = 8."""
    w = np.array([-0.75, -0.3, 0.0, 0.3, 0.75], np.float32)
    s, z = qz.asym_params(w.min(), w.max(), 4)
    assert abs(float(s) - 0.1) < 1e-7
    assert float(z) == 8.0
    code = qz.quantize(w, s, z, 4)
    assert code.tolist() == [0, 5, 8, 11, 15]
    np.testing.assert_allclose(qz.dequantize(code, s, z), [-0.8, -0.3, 0.0, 0.3, 0.7], atol=1e-6)


def test_asym_zero_point_derivation():
    """[Q-INT8] §Deriving the scale and zero-point: x_min -> q_min, x_max -> q_max (no clamping
    of z): s = (x_max - x_min)/(q_max - q_min), z = round(q_min - x_min/s)."""
    rng = np.random.default_rng(0)
    lo = -rng.uniform(0.01, 1.0, 2000)
    hi = rng.uniform(0.01, 1.0, 2000)
    for bits in (3, 4, 8):
        s, z = qz.asym_params(lo, hi, bits)
        np.testing.assert_allclose(s, (hi - lo) / (2 ** bits - 1), rtol=1e-15)
        assert np.all(qz.quantize(lo, s, z, bits) == 0)
        assert np.all(qz.quantize(hi, s, z, bits) == 2 ** bits - 1)


def test_rounding_error_at_most_half_step():
    """Inside [min, max], |w - w_hat| <= s/2 up to the zero-point rounding (<= s)."""
    rng = np.random.default_rng(1)
    W = rng.normal(0, 0.02, (64, 128))
    for bits in (3, 4):
        s, z = qz.params_from_values(W, bits, False)
        code = qz.quantize(W, s[:, None], z[:, None], bits)
        err = np.abs(W - qz.dequantize(code, s[:, None], z[:, None]))
        assert np.all(err <= s[:, None] * (0.5 + 1e-9) + s[:, None] * 0.5)
        # away from the clamped ends the half-step bound is exact
        inner = (code > 0) & (code < 2 ** bits - 1)
        assert np.all(err[inner] <= (s[:, None] * 0.5 * (1 + 1e-9)).repeat(128, 1)[inner])


def test_symmetric_range_and_zero():
    """[INT4-GPTQ] §Uniform INT4: symmetric q in [-2^(b-1), 2^(b-1)-1], s = max|w|/(2^(b-1)-1)."""
    rng = np.random.default_rng(2)
    W = rng.normal(0, 1, (32, 64)).astype(np.float32)
    s, z = qz.params_from_values(W, 4, True)
    np.testing.assert_array_equal(s, np.max(np.abs(W), 1) / np.float32(7))
    assert np.all(z == 8)
    code = qz.quantize(W, s[:, None], z[:, None], 4)
    q = code - 8
    assert q.min() >= -7 and q.max() <= 7                    # |w/s| <= 7 by construction
    assert np.all(np.abs(q).max(axis=1) == 7)                # the max-magnitude weight hits 7


def test_degenerate_group_uses_unit_scale():
    """A constant group (max == min) uses s = 1; an all-zero group decodes to zero."""
    s, z = qz.asym_params(np.float32(0), np.float32(0), 4)
    assert float(s) == 1.0 and float(z) == 0.0
    code = qz.quantize(np.zeros(4, np.float32), s, z, 4)
    assert np.all(qz.dequantize(code, s, z) == 0)
    s, z = qz.sym_params(np.float32(0), 4)
    assert float(s) == 1.0


def test_round_half_to_even():
    """Round-half-to-even (the rounding of the pages' tensor code): 0.5 -> 0, 1.5 -> 2, 2.5 -> 2."""
    w = np.array([0.5, 1.5, 2.5, -0.5, -1.5], np.float32)
    code = qz.quantize(w, np.float32(1), np.float32(8), 4)
    assert (code - 8).tolist() == [0, 2, 2, 0, -2]


@pytest.mark.parametrize("sym", [False, True])
def test_rtn_float32_matches_float64_off_ties(sym):
    """RTN in float32 and float64 agree except on codes whose w/s lies within 1e-5 of a tie."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (128, 256)).astype(np.float32)
    c32, s32, z32 = qz.rtn(W, 4, 128, sym)
    c64, s64, z64 = qz.rtn(W.astype(np.float64), 4, 128, sym)
    np.testing.assert_allclose(s32, s64, rtol=1e-6)
    frac = np.abs((W / np.repeat(s64, 128, 1)) % 1 - 0.5)
    near_tie = frac < 1e-5
    assert np.all((c32 == c64) | near_tie)
