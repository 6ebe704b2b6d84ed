"""Pins for oracle/gemv.py (no GPU)."""
import numpy as np

from conftest import parse_matrix, read_golden
from oracle import error as er
from oracle import gemv as gv
from oracle import pack as pk


def test_hand_case():
    g = read_golden("gemv_hand.txt")
    words = np.array([[int(w, 16) for w in row] for row in parse_matrix(g["words"], str)],
                     np.uint32)
    codes = np.array(parse_matrix(g["codes"], int), np.uint8)
    s = np.array(parse_matrix(g["scales"]), np.float32)
    z = np.array(parse_matrix(g["zeros"]), np.float32)
    x = np.array([float(t) for t in g["x"].split()])
    y = np.array([float(t) for t in g["y"].split()])
    qw, s16, z16 = pk.pack(codes, s, z, 4)
    np.testing.assert_array_equal(qw, words)
    got = gv.dequant_gemv(qw, s16, z16, np.zeros(8, np.int64), 8, 4, x)
    np.testing.assert_array_equal(got[0], y)


def test_matches_direct_dequantization_all_widths():
    """Through the packed words == from the codes directly, for every bit width and a
    permuted g_idx (act-order)."""
    rng = np.random.default_rng(2)
    n, d, g = 24, 256, 32
    for bits in (2, 3, 4, 8):
        codes = rng.integers(0, 2 ** bits, (n, d)).astype(np.uint8)
        S = rng.uniform(0.001, 0.05, (n, d // g)).astype(np.float32)
        Z = rng.integers(0, 2 ** bits, (n, d // g)).astype(np.float32)
        g_idx = rng.permutation(d) // g
        X = rng.normal(0, 1, (3, d)).astype(np.float16).astype(np.float64)
        qw, s16, z16 = pk.pack(codes, S, Z, bits)
        y = gv.dequant_gemv(qw, s16, z16, g_idx, d, bits, X)
        S16 = gv.fp16_bits_to_f64(s16)
        Z16 = gv.fp16_bits_to_f64(z16)
        ref = X @ er.dequant_matrix(codes, S16, Z16, g_idx).T
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_linear_in_x():
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 16, (8, 64)).astype(np.uint8)
    qw, s16, z16 = pk.pack(codes, np.full((8, 2), 0.01, np.float32),
                           np.full((8, 2), 8, np.float32), 4)
    gi = np.arange(64) // 32
    a, b = rng.normal(size=64), rng.normal(size=64)
    ya = gv.dequant_gemv(qw, s16, z16, gi, 64, 4, a)
    yb = gv.dequant_gemv(qw, s16, z16, gi, 64, 4, b)
    np.testing.assert_allclose(gv.dequant_gemv(qw, s16, z16, gi, 64, 4, 2 * a - 3 * b),
                               2 * ya - 3 * yb, rtol=1e-12, atol=1e-12)
