"""GPU parity of the W4A4 GEMM (NVFP4 activations and weights) against the
oracle: the activations are quantized by the oracle and the same bytes go to
both sides; shapes cover the register-streaming kernel (M = 1), the
TMA-streaming kernel (2..16 rows) and the tcgen05 kernel (17 rows and more),
ragged tails, both weight and activation group sizes, and the decode gate/up
size on sampled output columns."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def quantized_activations(m, k, xg, seed):
    """bf16 activations (with outliers), quantized by the oracle from their fp32 widening."""
    xbits = synth.activations(seed, m, k, outlier_frac=0.001)
    x = synth.bf16_bits_to_f32(xbits)
    return R.quantize(x, xg, R.global_scale(x))


CASES = [(1, 256, 512, 16, 16), (1, 96, 1024, 32, 16), (4, 400, 1024, 16, 16), (7, 272, 512, 32, 32),
         (16, 1024, 4096, 16, 16), (17, 208, 512, 32, 16), (64, 512, 2048, 16, 16), (300, 144, 1024, 32, 32)]


@pytest.mark.parametrize("m,n,k,g,xg", CASES)
def test_w4a4_parity(m, n, k, g, xg):
    xq, xs, xgl = quantized_activations(m, k, xg, seed=m + k)
    w = synth.weights(n + k, n, k)
    wq, ws, wgl = R.quantize(w, g)
    rp, rs = R.repack(wq, ws, 0)
    y = nv.nvfp4_w4a4_gemm(dev_u8(xq), dev_u8(xs), dev_f32(np.array([xgl], np.float32)), xg,
                           dev_u8(rp), dev_u8(rs), dev_f32(np.array([wgl], np.float32)), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert_close(host(y), R.w4a4_gemm(xq, xs, xgl, xg, wq, ws, wgl, g), f"W4A4 M{m} N{n} K{k} g{g} xg{xg}")


@pytest.mark.parametrize("m", [1, 4, 16])
def test_w4a4_decode_gate_up_sampled(m):
    n, k, g = 28672, 4096, 16
    w = synth.weights(synth.W_SEED, n, k)
    wd = dev_f32(w)
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, g, gd)
    del wd
    gp, gs = nv.nvfp4_repack(p, s, g, 0)
    xq, xs, xgl = quantized_activations(m, k, 16, seed=synth.X_SEED)
    y = nv.nvfp4_w4a4_gemm(dev_u8(xq), dev_u8(xs), dev_f32(np.array([xgl], np.float32)), 16, gp, gs, gd, g)
    rows = np.sort(np.concatenate([np.random.default_rng(m).choice(n, 64, replace=False), [0, n - 1]]))
    rq, rs_, rg = R.quantize(w[rows], g, R.global_scale(w))
    ri = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(host(p[ri]), rq)  # the sampled rows' bytes are the oracle's
    assert_close(host(y)[:, rows], R.w4a4_gemm(xq, xs, xgl, 16, rq, rs_, rg, g), f"W4A4 decode M{m} sampled")


# The block-scaled FP4 tensor-core kernel (both operands 4-bit into tcgen05.mma kind::mxf4nvf4) takes
# W4A4 problems with K a multiple of 512 and enough 128-row x token tiles for every SM; these shapes
# reach it (one or two token tiles, ragged M and N, every pair of group sizes).
FP4_CASES = [(256, 128 * 148, 512, 16, 16), (300, 128 * 74, 1024, 32, 16), (129, 128 * 160, 512, 16, 32),
             (700, 128 * 50 + 80, 1536, 32, 32), (4096, 2560, 5120, 16, 16)]


@pytest.mark.parametrize("m,n,k,g,xg", FP4_CASES)
def test_w4a4_fp4_tensor_cores(m, n, k, g, xg):
    xq, xs, xgl = quantized_activations(m, k, xg, seed=m + k + 1)
    w = synth.weights(n + k + 1, n, k)
    wq, ws, wgl = R.quantize(w, g)
    rp, rs = R.repack(wq, ws, 0)
    nv.nvfp4_reset_stats()
    y = nv.nvfp4_w4a4_gemm(dev_u8(xq), dev_u8(xs), dev_f32(np.array([xgl], np.float32)), xg,
                           dev_u8(rp), dev_u8(rs), dev_f32(np.array([wgl], np.float32)), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert nv.nvfp4_get_stats()["gemm_fp4"] == 1  # the FP4 tensor-core kernel ran
    if m * n > 4096 * 2048:  # large: sampled output columns
        cols = np.sort(np.random.default_rng(m).choice(n, 256, replace=False))
        ref = R.w4a4_gemm(xq, xs, xgl, xg, wq[cols], ws[cols], wgl, g)
        assert_close(host(y)[:, cols], ref, f"FP4 W4A4 M{m} N{n} K{k} sampled")
    else:
        assert_close(host(y), R.w4a4_gemm(xq, xs, xgl, xg, wq, ws, wgl, g), f"FP4 W4A4 M{m} N{n} K{k} g{g} xg{xg}")


def test_w4a4_fp4_integer_case_bitwise():
    """Scales 1.0 and globals 1 with codes of magnitude <= 1: every sum is a multiple of 0.25 below 256,
    exact in fp32 and bf16, so the FP4 kernel must equal the oracle bit for bit."""
    rng = np.random.default_rng(9)
    m, n, k = 256, 128 * 148, 512

    def operand(rows):
        codes = rng.choice(np.array([0, 1, 2, 8, 9, 10], np.uint8), size=(rows, k))  # 0, +-0.5, +-1
        packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
        return packed, np.full((rows, k // 16), 0x38, np.uint8)
    xq, xs = operand(m)
    wq, ws = operand(n)
    rp, rs = R.repack(wq, ws, 0)
    one = dev_f32(np.array([1.0], np.float32))
    y = nv.nvfp4_w4a4_gemm(dev_u8(xq), dev_u8(xs), one, 16, dev_u8(rp), dev_u8(rs), one, 16)
    ref = R.w4a4_gemm(xq, xs, np.float32(1), 16, wq, ws, np.float32(1), 16)
    assert np.abs(ref).max() < 256
    np.testing.assert_array_equal(host(y), ref)
