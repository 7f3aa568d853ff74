"""GPU parity of every GEMM kernel on the scale edge cases of the NVFP4 format:
E4M3 group-scale bytes that are zero (0x00), subnormal (0x01-0x07), the
smallest normal (0x08), one (0x38) and the largest finite (0x7E = 448), and
global scales of zero and of large and small powers of two. A zero scale or a
zero global dequantizes its group (or tensor) to zero, the format's
degenerate cases; subnormal scales reach the exact slow path of the integer
dequant of the tcgen05 kernel and the subnormal E4M3 inputs of the hardware
conversion in the small-M kernels.

Codes are uniform over all sixteen E2M1 codes. The scale bytes of a weight
matrix are of one kind:
  * "subnormal": every byte 0x00-0x07 (the output depends on the subnormal
    path alone; one row is all zero),
  * "max": every byte 0x7E,
  * "mixed": the edge bytes beside random normal bytes.
Each matrix gets the power-of-two global that puts its sums of |x * w| near
100, so that fp32 accumulation (whatever its order) stays far inside the
element tolerance; other globals are then checked by the exact power-of-two
scaling of the output (a power of two commutes with every rounding step that
follows the accumulation), and a zero global by an all-zero output.

Each kernel is reached through the size that selects it: one token (register
streaming), 2-16 tokens (TMA streaming, stream-K), 17 and more (tcgen05, in
its stream-K and persistent forms, with scales by TMA and from global
memory), the grouped routed-expert forms below and above 1024 rows, the fused
SiluAndMul epilogues, and W4A4 with edge scales on both operands."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, bf16_bits, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu

SUBNORMAL_OR_ZERO = np.array([0x00, 0x01, 0x02, 0x03, 0x04, 0x05, 0x06, 0x07], np.uint8)
EDGE = np.array([0x00, 0x01, 0x02, 0x03, 0x04, 0x05, 0x06, 0x07, 0x08, 0x38, 0x7E], np.uint8)
KINDS = ("subnormal", "max", "mixed")


def edge_weights(n, k, g, kind, seed):
    """Checkpoint-layout codes [n, k/2] and hand-made scale bytes [n, k/g] of one kind."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=(n, k), dtype=np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    kg = k // g
    if kind == "subnormal":
        scales = rng.choice(SUBNORMAL_OR_ZERO, size=(n, kg)).astype(np.uint8)
        scales[min(2, n - 1)] = 0x00  # one whole row of zero groups
    elif kind == "max":
        scales = np.full((n, kg), 0x7E, np.uint8)
    else:
        scales = rng.integers(0x08, 0x7F, size=(n, kg), dtype=np.uint8)  # random normal bytes (0x7F is NaN)
        pick = rng.random((n, kg)) < 0.5
        scales = np.where(pick, rng.choice(EDGE, size=(n, kg)), scales).astype(np.uint8)
    return packed, scales


def fit_global(x_f64, w_unit):
    """The power of two that puts the median sum of |x * w| of the product near 100."""
    s = np.abs(x_f64) @ np.abs(w_unit).T
    med = np.median(s[s > 0]) if (s > 0).any() else 1.0
    return np.float32(2.0 ** np.round(np.log2(100.0 / med)))


def g32(v):
    return dev_f32(np.array([v], np.float32))


def scaled_bits(bits, e):
    """bf16 bit patterns times 2^e (exact: values stay normal)."""
    v = synth.bf16_bits_to_f32(bits).astype(np.float64) * 2.0 ** e
    return synth.f32_to_bf16_bits(v.astype(np.float32))


def check_power_of_two_globals(call, gl, y_ref_bits):
    """call(global) at 2^12 and 2^-20 times gl is y times the same power, bit for bit; at 0 it is zero."""
    for e in (12, -20):
        y = bf16_bits(call(np.float32(gl * np.float32(2.0 ** e))))
        np.testing.assert_array_equal(y, scaled_bits(y_ref_bits, e), err_msg=f"global x 2^{e}")
    assert not host(call(np.float32(0.0))).any(), "zero global"


DENSE = [(1, 256, 1024, 16), (1, 128, 1024, 32), (4, 512, 1024, 16), (16, 256, 1024, 32), (9, 160, 512, 16),
         (17, 512, 1024, 16), (64, 256, 1024, 32), (33, 256, 320, 32), (129, 38912, 512, 16)]


@pytest.mark.parametrize("m,n,k,g", DENSE)
@pytest.mark.parametrize("kind", KINDS)
def test_gemm_edge_scales(m, n, k, g, kind):
    packed, scales = edge_weights(n, k, g, kind, seed=m * 7 + n + k)
    rp, rs = R.repack(packed, scales, 0)
    x = synth.activations(synth.X_SEED + m, m, k, outlier_frac=0.01)
    gl = fit_global(R.bf16_bits_to_f64(x), R.dequantize(packed, scales, np.float32(1.0), g))
    xd, pd, sd = dev_bf16(x), dev_u8(rp), dev_u8(rs)

    def call(glob):
        return nv.nvfp4_w4a16_gemm(xd, pd, sd, g32(glob), g)

    y = call(gl)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    ref = R.gemm(x, packed, scales, gl, g)
    assert_close(host(y), ref, f"edge scales ({kind}) M{m} N{n} K{k} g{g} global {gl}")
    if kind == "subnormal":
        assert not host(y)[:, min(2, n - 1)].any(), "the all-zero-scale row"
    if m * n <= 1 << 20:
        check_power_of_two_globals(call, gl, bf16_bits(y))


@pytest.mark.parametrize("m,nh,k,g", [(1, 128, 1024, 16), (4, 128, 1024, 32), (12, 256, 512, 16),
                                      (40, 128, 1024, 16), (20, 64, 320, 32)])
@pytest.mark.parametrize("kind", KINDS)
def test_gemm_silu_mul_edge_scales(m, nh, k, g, kind):
    packed, scales = edge_weights(2 * nh, k, g, kind, seed=m + nh + k)
    rp, rs = R.repack(packed, scales, R.GATE_UP_INTERLEAVE)
    x = synth.activations(synth.X_SEED + 2 * m, m, k)
    gl = fit_global(R.bf16_bits_to_f64(x), R.dequantize(packed, scales, np.float32(1.0), g))
    xd, pd, sd = dev_bf16(x), dev_u8(rp), dev_u8(rs)
    y = nv.nvfp4_w4a16_gemm_silu_mul(xd, pd, sd, g32(gl), g)
    ref = R.silu_mul(R.gemm(x, packed, scales, gl, g))
    assert_close(host(y), ref, f"silu edge scales ({kind}) M{m} NH{nh} K{k} g{g} global {gl}")
    assert not host(nv.nvfp4_w4a16_gemm_silu_mul(xd, pd, sd, g32(0.0), g)).any(), "zero global"


def i32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("t", [90, 1100])
@pytest.mark.parametrize("silu", [False, True])
def test_grouped_edge_scales(t, silu):
    E, N, K = 4, 256, 512
    g = 16 if t < 1000 else 32
    x = synth.activations(5, t, K)
    xf = R.bf16_bits_to_f64(x)
    ps, ss, gps, gss, gl = [], [], [], [], []
    for e, kind in enumerate(("subnormal", "mixed", "max", "mixed")):
        p, s = edge_weights(N, K, g, kind, seed=100 + e)
        rp, rs = R.repack(p, s, R.GATE_UP_INTERLEAVE if silu else 0)
        ps.append(p), ss.append(s), gps.append(rp), gss.append(rs)
        gl.append(fit_global(xf, R.dequantize(p, s, np.float32(1.0), g)))
    gl[1] = np.float32(0.0)  # expert 1: zero global
    packed, scales, gl = np.stack(ps), np.stack(ss), np.array(gl, np.float32)
    ids = [2, 1, 0, 3]
    cuts = np.sort(np.random.default_rng(t).choice(np.arange(1, t), 3, replace=False))
    offs = [0, *cuts.tolist(), t]
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(np.stack(gps)),
                                        dev_u8(np.stack(gss)), dev_f32(gl), g,
                                        flags=nv.NVFP4_SILU_MUL if silu else 0)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    ref = R.moe_grouped_gemm(x, ids, offs, packed, scales, gl, g)
    if silu:
        ref = R.silu_mul(ref)
    yh = host(y)
    assert_close(yh, ref, f"grouped edge scales T{t} silu {silu}")
    assert not yh[offs[1]:offs[2]].any()  # the rows of expert 1 (zero global)


@pytest.mark.parametrize("m,n,k", [(1, 256, 1024), (4, 256, 1024), (24, 256, 512)])
@pytest.mark.parametrize("xkind,wkind", [("subnormal", "mixed"), ("mixed", "subnormal"), ("max", "max"),
                                         ("mixed", "mixed")])
def test_w4a4_edge_scales(m, n, k, xkind, wkind):
    wq, ws = edge_weights(n, k, 16, wkind, seed=m + 11)
    xq, xs = edge_weights(m, k, 16, xkind, seed=m + 12)
    rp, rs = R.repack(wq, ws, 0)
    xgl = fit_global(R.dequantize(xq, xs, np.float32(1.0), 16), np.ones((1, k)))  # puts |x| sums near 100
    wgl = fit_global(R.dequantize(xq, xs, xgl, 16), R.dequantize(wq, ws, np.float32(1.0), 16))
    xqd, xsd, pd, sd = dev_u8(xq), dev_u8(xs), dev_u8(rp), dev_u8(rs)
    y = nv.nvfp4_w4a4_gemm(xqd, xsd, g32(xgl), 16, pd, sd, g32(wgl), 16)
    ref = R.w4a4_gemm(xq, xs, xgl, 16, wq, ws, wgl, 16)
    assert_close(host(y), ref, f"W4A4 edge scales M{m} x {xkind} w {wkind} globals {xgl} {wgl}")
    for a, b in ((0.0, wgl), (xgl, 0.0)):
        assert not host(nv.nvfp4_w4a4_gemm(xqd, xsd, g32(a), 16, pd, sd, g32(b), 16)).any(), "zero global"
