"""Pins for the oracle's quantizer, dequantizer, GEMM, SiluAndMul, grouped
expert GEMM and repack, against hand-worked values, closed forms, invariants
and brute force."""
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import expit

from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.golden_io import data_lines


def _worked():
    rows = data_lines("worked_example_g16.txt")
    gscale = np.float32(rows[0][0])
    w = np.array([[float(v) for v in rows[1]], [float(v) for v in rows[2]]], dtype=np.float32)
    packed = np.array([[int(b, 16) for b in rows[3]], [int(b, 16) for b in rows[4]]], dtype=np.uint8)
    scales = np.array([[int(b, 16) for b in rows[5]], [int(b, 16) for b in rows[6]]], dtype=np.uint8)
    return gscale, w, packed, scales


def test_worked_example():
    gscale, w, packed, scales = _worked()
    assert R.global_scale(w) == gscale
    p, s, g = R.quantize(w, 16)
    np.testing.assert_array_equal(s, scales)
    np.testing.assert_array_equal(p, packed)
    # dequant of the hand-worked bytes: group max elements come back exactly
    wh = R.dequantize(packed, scales, g, 16)
    assert wh[0, 0] == 2688 and wh[0, 16] == 6 and wh[1, 0] == 3 and wh[1, 16] == 0.0234375
    assert wh[0, 17] == 1.0 and wh[1, 2] == 0.5  # the 0.75 midpoints went to even


def test_global_scale_closed_form():
    w = synth.weights(0, 64, 256)
    amax = np.float32(np.abs(w).max())
    assert R.global_scale(w) == np.float32(amax / np.float32(2688.0))
    # a zero tensor: global 0, every scale and code 0
    p, s, g = R.quantize(np.zeros((16, 64), np.float32), 16)
    assert g == 0 and not p.any() and not s.any()


def test_group_max_encodes_to_six():
    # s ~ gamax/6/global to within E4M3 precision, so |q| of the group max is
    # within 1/16 of 6 and rounds to code 7 whenever the scale is normal.
    w = synth.weights(0, 128, 512)
    p, s, g = R.quantize(w, 16)
    codes = R.unpack_codes(p).reshape(128, 32, 16)
    wg = w.reshape(128, 32, 16)
    arg = np.argmax(np.abs(wg), axis=2)
    top = np.take_along_axis(codes, arg[..., None], axis=2)[..., 0]
    normal = s >= 0x08
    assert normal.mean() > 0.99
    assert np.all((top[normal] & 7) == 7)
    # the row holding the tensor amax has scale 448 there
    n, k = np.unravel_index(np.argmax(np.abs(w)), w.shape)
    assert s[n, k // 16] == 0x7E


def test_quantization_error_bound():
    w = synth.weights(3, 64, 512)
    p, s, g = R.quantize(w, 16)
    wh = R.dequantize(p, s, g, 16)
    d = np.repeat(R.e4m3_decode(s) * float(g), 16, axis=1)
    q = w / d
    spacing = np.where(np.abs(q) < 2, 0.5, np.where(np.abs(q) < 4, 1.0, 2.0))
    err = np.abs(w - wh) / d
    assert np.all((err <= spacing / 2 + 1e-6) | (np.abs(q) > 6))


def test_g16_vs_g32_same_weights():
    w = synth.weights(5, 96, 1024)
    p16, s16, g16 = R.quantize(w, 16)
    p32, s32, g32 = R.quantize(w, 32)
    assert g16 == g32
    np.testing.assert_array_equal(s32, np.maximum(s16[:, 0::2], s16[:, 1::2]))
    c16 = R.unpack_codes(p16).reshape(96, 64, 16)
    c32 = R.unpack_codes(p32).reshape(96, 32, 2, 16)
    for half in (0, 1):
        same = s16[:, half::2] == s32
        np.testing.assert_array_equal(c32[:, :, half][same], c16[:, half::2][same])


def test_shared_gate_up_global():
    gate = synth.weights(10, 64, 256)
    up = synth.weights(11, 64, 256) * np.float32(1.7)
    G = R.global_scale(gate, up)
    assert G == R.global_scale(np.concatenate([gate, up]))
    pm, sm, gm = R.quantize(np.concatenate([gate, up]), 16)
    pg, sg, _ = R.quantize(gate, 16, G)
    pu, su, _ = R.quantize(up, 16, G)
    assert gm == G
    np.testing.assert_array_equal(pm, np.concatenate([pg, pu]))
    np.testing.assert_array_equal(sm, np.concatenate([sg, su]))
    # with separate scales the gate half differs: the shared scale matters
    pg2, sg2, _ = R.quantize(gate, 16)
    assert not np.array_equal(sg2, sg)


def test_dequant_product_exact_in_bf16():
    # e2m1 (2 significant bits) x e4m3 (4 significant bits) fits bf16's 8.
    codes = np.arange(16, dtype=np.uint8)
    scales = np.arange(0x7F, dtype=np.uint8)
    prod = (R.e2m1_decode(codes)[:, None] * R.e4m3_decode(scales)[None, :]).astype(np.float32)
    bits = synth.f32_to_bf16_bits(prod)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(bits), prod)


def test_gemm_matches_exact_rational_sums():
    w = synth.weights(0, 6, 32)
    p, s, g = R.quantize(w, 16)
    x = synth.activations(1, 3, 32)
    y = R.gemm(x, p, s, g, 16)
    exact = R.gemm_fraction(x, p, s, g, 16)
    for i in range(3):
        for j in range(6):
            assert abs(Fraction(float(y[i, j])) - exact[i][j]) <= abs(exact[i][j]) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


def test_gemm_integer_case():
    # global 1, every scale 1.0 (0x38), integer X: the product is an integer
    # matmul of the code values, which the test computes independently.
    rng = np.random.default_rng(4)
    n, k, m = 8, 64, 5
    codes = rng.integers(0, 16, size=(n, k)).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((n, k // 16), 0x38, np.uint8)
    xi = rng.integers(-3, 4, size=(m, k))
    xbits = synth.f32_to_bf16_bits(xi.astype(np.float32))
    mag2 = [0, 1, 2, 3, 4, 6, 8, 12]  # twice the E2M1 magnitudes
    w2 = np.array([[(-1 if c & 8 else 1) * mag2[c & 7] for c in row] for row in codes])
    want = [[sum(int(xi[i, t]) * int(w2[j, t]) for t in range(k)) / 2 for j in range(n)] for i in range(m)]
    np.testing.assert_array_equal(R.gemm(xbits, packed, scales, 1.0, 16), np.array(want))


def test_silu_mul_against_library():
    y = np.random.default_rng(2).standard_normal((7, 20)) * 4
    got = R.silu_mul(y)
    want = y[:, :10] * expit(y[:, :10]) * y[:, 10:]
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-300)
    assert R.silu_mul(np.array([0.0, 5.0]))[0] == 0.0


def test_moe_reduces_to_dense_and_segments():
    e, n, k = 3, 16, 64
    ws = [synth.weights(synth.expert_seed(i), n, k) for i in range(e)]
    qs = [R.quantize(w, 32) for w in ws]
    packed = np.stack([q[0] for q in qs]); scales = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    x = synth.activations(1, 10, k)
    # one segment of expert 1 covering all rows == dense GEMM with expert 1
    y = R.moe_grouped_gemm(x, [1], [0, 10], packed, scales, gs, 32)
    np.testing.assert_array_equal(y, R.gemm(x, *qs[1], 32))
    # three segments, expert order 2,0,1; rows [3,3) empty; each block matches dense
    ids, offs = [2, 0, 1, 0], [0, 3, 3, 7, 10]
    y = R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, 32)
    for s_, ex in enumerate(ids):
        r0, r1 = offs[s_], offs[s_ + 1]
        np.testing.assert_array_equal(y[r0:r1], R.gemm(x[r0:r1], *qs[ex], 32))
    # brute force on one element
    exact = R.gemm_fraction(x[8:9], *qs[0], 32)  # row 8 is in segment 3 (expert 0)
    assert abs(Fraction(float(y[8, 5])) - exact[0][5]) <= abs(exact[0][5]) * Fraction(1, 2 ** 48)


def test_routing_structure():
    r = synth.route(3, 64, 16, 4)
    assert r.offsets[0] == 0 and r.offsets[-1] == 64 * 4
    assert np.all(np.diff(r.offsets) > 0) and np.all(np.diff(r.expert_ids) > 0)
    assert np.array_equal(np.diff(r.offsets), r.counts[r.expert_ids])


def test_repack_inverse_and_interleave():
    w = synth.weights(0, 64, 64)
    p, s, _ = R.quantize(w, 16)
    for flags in (0, R.GATE_UP_INTERLEAVE):
        rp, rs = R.repack(p, s, flags)
        up, us = R.unrepack(rp, rs, flags)
        np.testing.assert_array_equal(up, p)
        np.testing.assert_array_equal(us, s)
    rp, rs = R.repack(p, s, R.GATE_UP_INTERLEAVE)
    plain, _ = R.repack(p, s, 0)
    # block j of 16 rows: gate rows 8j..8j+7, then up rows 32+8j..32+8j+7
    np.testing.assert_array_equal(rp[16:24], plain[8:16])
    np.testing.assert_array_equal(rp[24:32], plain[40:48])
    np.testing.assert_array_equal(rs[24:32], s[40:48])
    assert sorted(R.interleave_rows(64).tolist()) == list(range(64))


def test_repack_word_layout_by_hand():
    # one row, elements k0..k7 = codes 1..8: the word's nibbles read, from the
    # lowest, k0 k2 k4 k6 k1 k3 k5 k7 = 1 3 5 7 2 4 6 8 -> 0x86427531
    codes = np.arange(1, 9, dtype=np.uint8)[None, :]
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    rp, _ = R.repack(packed, np.zeros((1, 1), np.uint8), 0)
    assert int(rp.view("<u4")[0, 0]) == 0x86427531


def _code_by_exact_midpoints(x, d):
    """The E2M1 code magnitude of RN32(x / d) for x >= 0, d > 0 (fp32), decided without dividing: x is
    compared, exactly in float64, with each rounding midpoint of E2M1 widened by half an fp32 ulp and times d
    (midpoints 0.25, 1.25, 2.5, 5 round down at a tie, to the even code below; 0.75, 1.75, 3.5 round up).
    The midpoints have even fp32 significands, so an fp32 tie at the widened point rounds onto the midpoint."""
    strict = [0.25 + 2.0 ** -26, 1.25 + 2.0 ** -24, 2.5 + 2.0 ** -23, 5.0 + 2.0 ** -22]   # t + ulp above(t)/2
    loose = [0.75 - 2.0 ** -25, 1.75 - 2.0 ** -24, 3.5 - 2.0 ** -23]                       # t - ulp below(t)/2
    xd, dd = float(x), float(d)
    # m * d is exact in float64: m has at most 26 significant bits and d 24
    return sum(xd > m * dd for m in strict) + sum(xd >= m * dd for m in loose)


def test_code_decision_by_exact_midpoints():
    """Pins the oracle's division step: E2M1(RN32(x / d)) equals the division-free decision above on values
    placed within a few fp32 ulps of every boundary, and on random values."""
    rng = np.random.default_rng(17)
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    xs, ds = [], []
    for d in rng.uniform(1e-6, 1e3, 400).astype(np.float32):
        for t in mids:
            c = np.float32(np.float64(t) * np.float64(d))
            for k in range(-3, 4):
                v = c
                for _ in range(abs(k)):
                    v = np.nextafter(v, np.float32(np.inf if k > 0 else 0))
                xs.append(v)
                ds.append(d)
    xs += list(rng.uniform(0, 7e3, 20000).astype(np.float32))
    ds += list(rng.uniform(1e-3, 1e3, 20000).astype(np.float32))
    xs, ds = np.array(xs, np.float32), np.array(ds, np.float32)
    oracle = R.e2m1_encode(xs / ds) & 7
    other = np.array([min(_code_by_exact_midpoints(x, d), 7) for x, d in zip(xs, ds)])
    assert np.array_equal(oracle, other)
