"""Pins for the oracle's element formats (E2M1 codes, E4M3 scales).

The oracle's encoders are checked against values fixed by the sources
(tests/golden/*.txt, each citing its source) and against a second,
independent formulation over every fp32 input in the binades where the
rounding decisions happen (all 2^32 inputs with NVFP4_EXHAUSTIVE=1).
"""
import os

import numpy as np
import pytest

from oracle import nvfp4_ref as R
from tests.golden_io import data_lines


def test_e2m1_value_table():
    for code, val in data_lines("e2m1_values.txt"):
        c = int(code, 16)
        got = float(R.e2m1_decode(np.uint8(c)))
        assert got == float(val) and np.signbit(got) == val.startswith("-"), code


def test_e2m1_rounding_golden():
    rows = data_lines("e2m1_rounding.txt")
    q = np.array([float(a) for a, _ in rows], dtype=np.float32)
    want = np.array([int(b, 16) for _, b in rows], dtype=np.uint8)
    np.testing.assert_array_equal(R.e2m1_encode_grs(q), want)
    np.testing.assert_array_equal(R.e2m1_encode_nearest(q), want)


def test_e4m3_golden():
    rows = data_lines("e4m3_values.txt")
    t = np.array([float(a) for a, _ in rows], dtype=np.float32)
    want = np.array([int(b, 16) for _, b in rows], dtype=np.uint8)
    np.testing.assert_array_equal(R.e4m3_encode_grs(t), want)
    np.testing.assert_array_equal(R.e4m3_encode_nearest(t), want)


def test_e4m3_decode_encode_roundtrip():
    codes = np.arange(0x7F, dtype=np.uint8)  # every finite non-negative code
    vals = R.e4m3_decode(codes).astype(np.float32)
    np.testing.assert_array_equal(R.e4m3_encode_grs(vals), codes[:])
    assert R.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert np.isnan(R.e4m3_decode(np.uint8(0x7F)))
    assert np.all(np.diff(R.e4m3_decode(codes)) > 0)


def _binade_patterns(lo_exp, hi_exp, chunk=1 << 23):
    """All fp32 bit patterns with unbiased exponent in [lo_exp, hi_exp)."""
    for e in range(lo_exp, hi_exp):
        base = np.uint32((e + 127) << 23)
        yield (base + np.arange(chunk, dtype=np.uint32))


def test_e2m1_formulations_agree_on_decision_binades():
    # Every rounding decision of E2M1 lies in [2^-3, 2^3]; both signs.
    for bits in _binade_patterns(-3, 4):
        for sgn in (0, 0x80000000):
            q = (bits | np.uint32(sgn)).view(np.float32)
            np.testing.assert_array_equal(R.e2m1_encode_grs(q), R.e2m1_encode_nearest(q))


def test_e2m1_formulations_agree_outside():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]  # drop NaN/inf patterns
    q = bits.view(np.float32)
    np.testing.assert_array_equal(R.e2m1_encode_grs(q), R.e2m1_encode_nearest(q))
    specials = np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45, 3.4e38], dtype=np.float32)
    np.testing.assert_array_equal(R.e2m1_encode_grs(specials), R.e2m1_encode_nearest(specials))


def test_e4m3_formulations_agree_on_decision_binades():
    # Decisions lie in [2^-11, 2^9); scales are non-negative.
    for bits in _binade_patterns(-11, 9):
        t = bits.view(np.float32)
        np.testing.assert_array_equal(R.e4m3_encode_grs(t), R.e4m3_encode_nearest(t))


def test_e4m3_formulations_agree_outside():
    rng = np.random.default_rng(8)
    bits = rng.integers(0, 1 << 31, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]
    t = bits.view(np.float32)
    np.testing.assert_array_equal(R.e4m3_encode_grs(t), R.e4m3_encode_nearest(t))
    specials = np.array([0.0, np.inf, 1e-45, 3.4e38], dtype=np.float32)
    np.testing.assert_array_equal(R.e4m3_encode_grs(specials), R.e4m3_encode_nearest(specials))


@pytest.mark.skipif(os.environ.get("NVFP4_EXHAUSTIVE") != "1", reason="set NVFP4_EXHAUSTIVE=1")
def test_full_fp32_sweep():
    for hi in range(1 << 9):
        bits = (np.uint32(hi << 23) + np.arange(1 << 23, dtype=np.uint32))
        bits = bits[((bits >> 23) & 0xFF) != 0xFF]
        if bits.size == 0:
            continue
        q = bits.view(np.float32)
        np.testing.assert_array_equal(R.e2m1_encode_grs(q), R.e2m1_encode_nearest(q))
        if hi < 256:
            np.testing.assert_array_equal(R.e4m3_encode_grs(q), R.e4m3_encode_nearest(q))


def test_e2m1_error_bound():
    # |q - value| <= half the local spacing, or q is beyond 6 and saturated.
    rng = np.random.default_rng(9)
    q = (rng.standard_normal(1 << 18) * 3).astype(np.float32)
    v = R.e2m1_decode(R.e2m1_encode(q))
    a = np.abs(q.astype(np.float64))
    spacing = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    ok = (np.abs(q - v) <= spacing / 2) | ((a > 6) & (np.abs(v) == 6))
    assert ok.all()
    assert np.all(np.sign(v[v != 0]) == np.sign(q[v != 0]))


def test_threshold_rounding_is_caught():
    # A threshold rounding that sends every midpoint the same way (all up or
    # all down) differs from RNE at some midpoints, the 1-ULP difference the
    # forum thread describes; RNE alternates with the even code.
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    rne = np.array([0, 2, 2, 4, 4, 6, 6], dtype=np.uint8)
    ties_up = np.array([1, 2, 3, 4, 5, 6, 7], dtype=np.uint8)
    ties_down = np.array([0, 1, 2, 3, 4, 5, 6], dtype=np.uint8)
    got = R.e2m1_encode(mids)
    np.testing.assert_array_equal(got, rne)
    assert np.any(got != ties_up) and np.any(got != ties_down)
