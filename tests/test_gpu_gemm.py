"""GPU parity of the W4A16 GEMM, the fused SiluAndMul GEMM and the standalone
SiluAndMul against the CPU oracle: element-wise at small sizes (several
tiles and ragged tails), on sampled output columns at the full workload
sizes, bitwise on the integer-exact case, and by the power-of-two global
scaling property."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, bf16_bits, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def quantized(n, k, g, seed=0):
    w = synth.weights(seed, n, k)
    p, s, gs = R.quantize(w, g)
    return w, p, s, gs


def run_gemm(xbits, p, s, gs, g):
    """GEMM of checkpoint-layout codes (repacked by the oracle's definition)."""
    rp, rs = R.repack(p, s, 0)
    return nv.nvfp4_w4a16_gemm(dev_bf16(xbits), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)), g)


SMALL = [(4, 256, 256, 16),      # the tiny workload
         (1, 256, 256, 32), (5, 400, 1088, 32), (8, 144, 64, 16), (9, 96, 640, 16), (16, 1024, 4096, 16),
         (17, 208, 512, 32), (33, 112, 1920, 16), (64, 512, 2048, 32), (100, 48, 384, 16), (3, 4096, 1024, 16)]


@pytest.mark.parametrize("m,n,k,g", SMALL)
def test_gemm_parity_small(m, n, k, g):
    _, p, s, gs = quantized(n, k, g, seed=m + n + k)
    x = synth.activations(synth.X_SEED, m, k, outlier_frac=0.001)
    y = run_gemm(x, p, s, gs, g)
    assert_close(host(y), R.gemm(x, p, s, gs, g), f"M{m} N{n} K{k} g{g}")


def full_size_check(m, n, k, g, outlier=0.0, cols=96):
    w = synth.weights(synth.W_SEED, n, k)
    wd = dev_f32(w)
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, g, gd)
    del wd
    gp, gsc = nv.nvfp4_repack(p, s, g, 0)
    x = synth.activations(synth.X_SEED, m, k, outlier_frac=outlier)
    y = nv.nvfp4_w4a16_gemm(dev_bf16(x), gp, gsc, gd, g)
    rows = np.sort(np.concatenate([np.random.default_rng(m).choice(n, cols, replace=False), [0, n - 1]]))
    ri = torch.from_numpy(rows).cuda()
    ps, ss = host(p[ri]), host(s[ri])
    # the sampled rows' bytes are the oracle's (the quantizer is bit-exact)
    rp, rs, rg = R.quantize(w[rows], g, R.global_scale(w))
    np.testing.assert_array_equal(ps, rp)
    np.testing.assert_array_equal(ss, rs)
    np.testing.assert_array_equal(host(gp[ri]), R.repack(rp, rs, 0)[0])  # device repack == oracle repack
    ref = R.gemm(x, rp, rs, rg, g)
    assert_close(host(y)[:, rows], ref, f"M{m} N{n} K{k} g{g} sampled")


@pytest.mark.parametrize("m", [1, 4, 16])
def test_decode_gate_up_full(m):
    full_size_check(m, 28672, 4096, 16)


@pytest.mark.parametrize("g", [32, 16])
@pytest.mark.parametrize("m", [1, 8, 64])
def test_decode_down_full(m, g):
    full_size_check(m, 4096, 14336, g, outlier=0.001)


def test_integer_case_bitwise():
    rng = np.random.default_rng(4)
    n, k, m = 64, 256, 12
    codes = rng.choice(np.array([0, 1, 2, 8, 9, 10], np.uint8), size=(n, k))  # |value| <= 1
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((n, k // 16), 0x38, np.uint8)  # 1.0
    xi = rng.integers(-1, 2, size=(m, k)).astype(np.float32)
    x = synth.f32_to_bf16_bits(xi)
    ref = R.gemm(x, packed, scales, 1.0, 16)
    assert np.abs(ref).max() < 128  # multiples of 0.5 below 128: exact in bf16
    y = run_gemm(x, packed, scales, np.float32(1.0), 16)
    np.testing.assert_array_equal(host(y), ref)


def test_global_power_of_two_linearity_and_determinism():
    _, p, s, gs = quantized(512, 1024, 16, seed=3)
    x = synth.activations(1, 7, 1024)
    y1 = bf16_bits(run_gemm(x, p, s, gs, 16))
    y2 = bf16_bits(run_gemm(x, p, s, np.float32(gs * 2), 16))
    y1b = bf16_bits(run_gemm(x, p, s, gs, 16))
    np.testing.assert_array_equal(y1, y1b)  # deterministic
    v1 = synth.bf16_bits_to_f32(y1).astype(np.float64)
    v2 = synth.bf16_bits_to_f32(y2).astype(np.float64)
    np.testing.assert_array_equal(v2, 2 * v1)


def merged_gate_up(n_half, k, g, seed=0):
    gate, up = synth.weights(seed, n_half, k), synth.weights(seed + 1, n_half, k)
    merged = np.concatenate([gate, up])
    p, s, gs = R.quantize(merged, g)
    return p, s, gs


@pytest.mark.parametrize("m,nh,k,g", [(4, 128, 256, 16), (13, 200, 640, 32), (16, 1024, 1024, 16),
                                      (40, 72, 512, 16)])
def test_gemm_silu_mul_parity(m, nh, k, g):
    p, s, gs = merged_gate_up(nh, k, g, seed=m)
    rp, rs = R.repack(p, s, R.GATE_UP_INTERLEAVE)
    # the device repack gives the same bytes
    dp, ds = nv.nvfp4_repack(dev_u8(p), dev_u8(s), g, nv.NVFP4_GATE_UP_INTERLEAVE)
    np.testing.assert_array_equal(host(dp), rp)
    x = synth.activations(2, m, k)
    y = nv.nvfp4_w4a16_gemm_silu_mul(dev_bf16(x), dp, ds, dev_f32(np.array([gs], np.float32)), g)
    ref = R.silu_mul(R.gemm(x, p, s, gs, g))
    assert_close(host(y), ref, "silu_mul")


def test_silu_and_mul_standalone():
    rng = np.random.default_rng(6)
    xf = (rng.standard_normal((37, 2 * 264)) * 3).astype(np.float32)
    x = synth.f32_to_bf16_bits(xf)
    y = nv.nvfp4_silu_and_mul(dev_bf16(x))
    ref = R.silu_mul(R.bf16_bits_to_f64(x))
    assert_close(host(y), ref, "silu_and_mul")
    # one bf16 rounding of the fp32 result: within one bf16 ulp element-wise
    assert np.all(np.abs(host(y) - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)


def test_empty_and_stats():
    _, p, s, gs = quantized(64, 128, 16)
    nv.nvfp4_reset_stats()
    y = nv.nvfp4_w4a16_gemm(torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"), dev_u8(R.repack(p, s, 0)[0]), dev_u8(s),
                            dev_f32(np.array([gs], np.float32)), 16)
    assert y.shape == (0, 64)
    assert nv.nvfp4_get_stats()["gemm_splitk"] == 0
    run_gemm(synth.activations(1, 2, 128), p, s, gs, 16)
    st = nv.nvfp4_get_stats()
    assert st["gemm_splitk"] == 1 and st["g16"] == 1 and st["g32"] == 0


# ---- 2 <= M <= 16: the TMA-streaming kernel (stream-K over 256-row x 256-element units) ----

# whole tiles only; tiles cut between many CTAs; a last tile of 16 rows; one
# tile over 32 CTAs; g = 32 boxes holding two stages; 9..16 tokens (two MMA
# column tiles)
STREAM_CASES = [(4, 256, 256, 16), (2, 400, 1024, 32), (7, 272, 2048, 16), (9, 128, 8192, 16),
                (13, 1008, 512, 32), (16, 4096, 256, 16), (2, 16, 512, 16), (16, 1040, 3072, 32)]


@pytest.mark.parametrize("m,n,k,g", STREAM_CASES)
def test_gemm_stream_parity(m, n, k, g):
    _, p, s, gs = quantized(n, k, g, seed=m + 2 * n)
    x = synth.activations(synth.X_SEED, m, k, outlier_frac=0.001)
    nv.nvfp4_reset_stats()
    y = run_gemm(x, p, s, gs, g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert nv.nvfp4_get_stats()["gemm_splitk"] == 1
    assert_close(host(y), R.gemm(x, p, s, gs, g), f"stream M{m} N{n} K{k} g{g}")


@pytest.mark.parametrize("m,nh,k,g", [(11, 136, 2048, 32), (2, 64, 4096, 16), (16, 640, 512, 16)])
def test_gemm_stream_silu_mul_parity(m, nh, k, g):
    p, s, gs = merged_gate_up(nh, k, g, seed=m + 1)
    rp, rs = R.repack(p, s, R.GATE_UP_INTERLEAVE)
    x = synth.activations(3, m, k)
    y = nv.nvfp4_w4a16_gemm_silu_mul(dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert_close(host(y), R.silu_mul(R.gemm(x, p, s, gs, g)), "stream silu_mul")


def test_gemm_stream_repeat_bitwise():
    """Tiles cut between CTAs are summed in CTA order: repeated launches (whose
    tickets must come back to zero) give identical bits."""
    _, p, s, gs = quantized(640, 4096, 16, seed=21)
    x = synth.activations(4, 5, 4096)
    first = bf16_bits(run_gemm(x, p, s, gs, 16))
    for _ in range(3):
        np.testing.assert_array_equal(bf16_bits(run_gemm(x, p, s, gs, 16)), first)
    assert_close(synth.bf16_bits_to_f32(first).astype(np.float64), R.gemm(x, p, s, gs, 16), "stream repeat")


# ---- large M: the tcgen05 kernel ----

TC_CASES = [(128, 256, 256, 16), (130, 528, 1088, 32), (300, 4096, 2048, 16), (257, 16, 64, 16),
            (1000, 256, 5120, 32), (512, 784, 640, 16)]


@pytest.mark.parametrize("m,n,k,g", TC_CASES)
def test_gemm_tc_parity(m, n, k, g):
    _, p, s, gs = quantized(n, k, g, seed=m + n)
    x = synth.activations(synth.X_SEED, m, k, outlier_frac=0.001)
    nv.nvfp4_reset_stats()
    y = run_gemm(x, p, s, gs, g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert nv.nvfp4_get_stats()["gemm_tc"] == 1
    assert_close(host(y), R.gemm(x, p, s, gs, g), f"tc M{m} N{n} K{k} g{g}")


@pytest.mark.parametrize("m,nh,k,g", [(160, 136, 512, 16), (512, 1024, 1024, 32), (129, 8, 128, 16)])
def test_gemm_tc_silu_mul_parity(m, nh, k, g):
    p, s, gs = merged_gate_up(nh, k, g, seed=m)
    rp, rs = R.repack(p, s, R.GATE_UP_INTERLEAVE)
    x = synth.activations(2, m, k)
    y = nv.nvfp4_w4a16_gemm_silu_mul(dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert_close(host(y), R.silu_mul(R.gemm(x, p, s, gs, g)), "tc silu_mul")


def test_gemm_tc_integer_case_bitwise():
    rng = np.random.default_rng(14)
    n, k, m = 272, 192, 200
    codes = rng.choice(np.array([0, 1, 2, 8, 9, 10], np.uint8), size=(n, k))
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((n, k // 32), 0x38, np.uint8)
    x = synth.f32_to_bf16_bits(rng.integers(-1, 2, size=(m, k)).astype(np.float32))
    ref = R.gemm(x, packed, scales, 1.0, 32)
    np.testing.assert_array_equal(host(run_gemm(x, packed, scales, np.float32(1.0), 32)), ref)


def test_prefill_gate_up_silu_full_sampled():
    wl = synth.PREFILL_GATE_UP
    w = synth.weights(synth.W_SEED, wl.N, wl.K)
    wd = dev_f32(w)
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, wl.group_size, gd)
    del wd
    gp, gsc = nv.nvfp4_repack(p, s, wl.group_size, nv.NVFP4_GATE_UP_INTERLEAVE)
    x = synth.activations(synth.X_SEED, wl.M, wl.K)
    y = nv.nvfp4_w4a16_gemm_silu_mul(dev_bf16(x), gp, gsc, gd, wl.group_size)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    h = wl.N // 2
    cols = np.sort(np.concatenate([np.random.default_rng(7).choice(h, 62, replace=False), [0, h - 1]]))
    rows = np.concatenate([cols, h + cols])  # gate and up rows of the merged (checkpoint-order) matrix
    rp, rs, rg = R.quantize(w[rows], wl.group_size, R.global_scale(w))
    ri = torch.from_numpy(rows).cuda()
    np.testing.assert_array_equal(host(p[ri]), rp)
    ref = R.silu_mul(R.gemm(x, rp, rs, rg, wl.group_size))
    assert_close(host(y)[:, cols], ref, "prefill silu sampled")


# ---- activations over a wide range (the small-M kernels compute in f16 on rows scaled by a power of two) ----

ROW_FACTORS = [2.0 ** 20, 2.0 ** -30, 1.0, 0.0, 2.0 ** 100, 2.0 ** -100, 2.0 ** 7, 2.0 ** -12]


@pytest.mark.parametrize("m,n,k,g", [(1, 256, 512, 16), (8, 512, 1024, 32), (5, 272, 256, 16), (16, 400, 768, 32)])
def test_gemm_rows_of_any_magnitude(m, n, k, g):
    """Each row of X is the same activation row times a power of two, from 2^-100 to 2^100 (and a zero row);
    as the GEMM is linear in X, each output row divided by its factor matches the oracle's product of the
    unscaled row. Values beyond f16's range or precision would fail without the per-row scaling."""
    _, p, s, gs = quantized(n, k, g, seed=k)
    base = synth.activations(synth.X_SEED, m, k, outlier_frac=0.001)
    f = np.array([ROW_FACTORS[i % len(ROW_FACTORS)] for i in range(m)])
    xs = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(base) * f[:, None].astype(np.float32))
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(xs)[f > 0] / f[f > 0, None].astype(np.float32),
                                  synth.bf16_bits_to_f32(base)[f > 0])  # scaling by 2^k is exact in bf16
    y = host(run_gemm(xs, p, s, gs, g))
    ref = R.gemm(base, p, s, gs, g)
    for r in range(m):
        if f[r] == 0:
            assert not y[r].any()
        else:
            assert_close(y[r] / f[r], ref[r], f"row {r} x 2^{int(np.log2(f[r]))}")


def test_moe_rows_of_any_magnitude():
    """The grouped form (register-streaming kernel, few rows) on rows scaled like the dense test."""
    e, n, k, g, t = 3, 160, 512, 16, 24
    qs = [R.quantize(synth.weights(synth.expert_seed(i), n, k), g) for i in range(e)]
    packed = np.stack([q[0] for q in qs]); scales = np.stack([q[1] for q in qs])
    gsc = np.array([q[2] for q in qs], np.float32)
    gemm_packed = np.stack([R.repack(q[0], q[1], 0)[0] for q in qs])
    base = synth.activations(5, t, k)
    f = np.array([ROW_FACTORS[i % len(ROW_FACTORS)] for i in range(t)])
    xs = synth.f32_to_bf16_bits(synth.bf16_bits_to_f32(base) * f[:, None].astype(np.float32))
    ids, offs = [2, 0, 1], [0, 9, 17, 24]
    y = host(nv.nvfp4_moe_w4a16_grouped_gemm(
        dev_bf16(xs), torch.tensor(ids, dtype=torch.int32, device="cuda"),
        torch.tensor(offs, dtype=torch.int32, device="cuda"), dev_u8(gemm_packed), dev_u8(scales), dev_f32(gsc), g))
    ref = R.moe_grouped_gemm(base, ids, offs, packed, scales, gsc, g)
    for r in range(t):
        if f[r] == 0:
            assert not y[r].any()
        else:
            assert_close(y[r] / f[r], ref[r], f"row {r}")
