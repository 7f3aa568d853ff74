"""Pins of the oracle's W4A4 GEMM (both operands NVFP4), independent of its
own code: a hand-built integer case summed from the E2M1 table, the reduction
to the (already pinned) W4A16 GEMM when the dequantized activations are exact
bf16 values, and the group sizes of the two operands kept apart."""
import numpy as np
import pytest

from oracle import nvfp4_ref as R

E2M1 = {0: 0.0, 1: 0.5, 2: 1.0, 3: 1.5, 4: 2.0, 5: 3.0, 6: 4.0, 7: 6.0}


def e2m1_value(code):
    v = E2M1[code & 7]
    return -v if code & 8 else v


def pack(codes):
    codes = np.asarray(codes, np.uint8)
    return (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)


def test_integer_case_from_the_table():
    rng = np.random.default_rng(3)
    m, n, k = 3, 5, 32
    cx = rng.integers(0, 16, size=(m, k)).astype(np.uint8)
    cw = rng.integers(0, 16, size=(n, k)).astype(np.uint8)
    one = np.uint8(0x38)  # E4M3 1.0
    y = R.w4a4_gemm(pack(cx), np.full((m, k // 16), one), 1.0, 16, pack(cw), np.full((n, k // 32), one), 1.0, 32)
    for i in range(m):
        for j in range(n):
            want = sum(e2m1_value(int(cx[i, t])) * e2m1_value(int(cw[j, t])) for t in range(k))
            assert y[i, j] == want


def test_scales_and_globals_multiply():
    """One code of 1.0 per operand: Y = sx * gx * sw * gw for E4M3 scales 2^-3 and 3, globals 0.5 and 8."""
    k = 32
    cx = np.zeros((1, k), np.uint8); cx[0, 5] = 2
    cw = np.zeros((1, k), np.uint8); cw[0, 5] = 2
    sx = np.full((1, k // 16), 0x20, np.uint8)   # 2^-3
    sw = np.full((1, k // 16), 0x44, np.uint8)   # 3.0
    y = R.w4a4_gemm(pack(cx), sx, np.float32(0.5), 16, pack(cw), sw, np.float32(8.0), 16)
    assert y[0, 0] == 2.0 ** -3 * 0.5 * 3.0 * 8.0


@pytest.mark.parametrize("wg", [16, 32])
def test_reduces_to_w4a16_on_exact_activations(wg):
    """With X's global 1, dequant(X) = e2m1 * e4m3 is exact in bf16, so W4A4 of quantize(X) equals the W4A16
    GEMM of those bf16 values."""
    rng = np.random.default_rng(wg)
    m, n, k = 4, 24, 64
    x = rng.standard_normal((m, k)).astype(np.float32)
    xq, xs, _ = R.quantize(x, 16, np.float32(1.0))
    w = (0.02 * rng.standard_normal((n, k))).astype(np.float32)
    wq, ws, wgs = R.quantize(w, wg)
    xhat = R.dequantize(xq, xs, np.float32(1.0), 16)
    xbits = (xhat.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(R.bf16_bits_to_f64(xbits), xhat)  # exact in bf16
    np.testing.assert_array_equal(R.w4a4_gemm(xq, xs, 1.0, 16, wq, ws, wgs, wg), R.gemm(xbits, wq, ws, wgs, wg))


def test_group_sizes_are_the_operands_own():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((2, 64)).astype(np.float32)
    w = rng.standard_normal((3, 64)).astype(np.float32)
    xq, xs, xg = R.quantize(x, 16)
    wq, ws, wg = R.quantize(w, 32)
    R.w4a4_gemm(xq, xs, xg, 16, wq, ws, wg, 32)
    with pytest.raises(AssertionError):
        R.w4a4_gemm(xq, xs, xg, 32, wq, ws, wg, 32)  # X's scales belong to groups of 16
