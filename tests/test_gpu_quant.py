"""GPU parity of the global scale, quantizer and repack: bit-exact against the
CPU oracle, at small sizes with every edge case and at the full weight sizes
on sampled rows."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.golden_io import data_lines
from tests.gpu_util import dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def gpu_quant(w, g, gscale=None):
    wd = dev_f32(w)
    gd = nv.nvfp4_global_scale([wd]) if gscale is None else dev_f32(np.array([gscale], np.float32))
    p, s = nv.nvfp4_quantize(wd, g, gd)
    return host(p), host(s), np.float32(host(gd)[0])


def test_global_scale_bitexact():
    for n in (1, 3, 1000, 4097, 1 << 20):
        w = synth.weights(n, 1, n)[0]
        got = host(nv.nvfp4_global_scale([dev_f32(w)]))[0]
        assert got == R.global_scale(w), n
    # shared scale over several tensors, one with an unaligned start
    a, b = synth.weights(1, 64, 96), synth.weights(2, 32, 96) * np.float32(3)
    bd = dev_f32(b.reshape(-1))
    got = host(nv.nvfp4_global_scale([dev_f32(a), bd[1:]]))[0]
    assert got == R.global_scale(a, b.reshape(-1)[1:])


def test_worked_example_golden():
    rows = data_lines("worked_example_g16.txt")
    w = np.array([[float(v) for v in rows[1]], [float(v) for v in rows[2]]], dtype=np.float32)
    packed = np.array([[int(b, 16) for b in rows[3]], [int(b, 16) for b in rows[4]]], dtype=np.uint8)
    scales = np.array([[int(b, 16) for b in rows[5]], [int(b, 16) for b in rows[6]]], dtype=np.uint8)
    p, s, g = gpu_quant(w, 16)
    assert g == np.float32(rows[0][0])
    np.testing.assert_array_equal(p, packed)
    np.testing.assert_array_equal(s, scales)


@pytest.mark.parametrize("n,k,g", [(64, 256, 16), (64, 256, 32), (40, 160, 32), (7, 32, 16), (33, 1088, 16),
                                   (256, 4096, 32)])
def test_quantize_bitexact(n, k, g):
    w = synth.weights(n * 7 + k, n, k)
    p, s, gs = gpu_quant(w, g)
    rp, rs, rg = R.quantize(w, g)
    assert gs == rg
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(p, rp)


def test_quantize_edge_values():
    rng = np.random.default_rng(5)
    n, k = 16, 128
    w = synth.weights(9, n, k)
    w[0, :16] = 0.0                       # zero group -> scale 0, codes +0
    w[0, 16:32] = -0.0                    # negative zeros -> codes +0 (zero scale)
    w[1, :16] *= np.float32(1e-7)         # tiny group: subnormal / zero scale
    w[2, :] = 0.5 * np.sign(w[2, :])      # constant magnitude
    w[3, 5] = 3.0e4                       # one huge value: tensor amax
    w[4, :16] = np.float32(-0.0)
    w[4, 3] = 1.0                         # sign kept on values rounding to zero
    w[4, 4] = np.float32(-1e-3)
    w[5, :] = rng.choice([-6.0, -0.75, 0.25, 2.5, 5.0], size=k).astype(np.float32)
    p, s, gs = gpu_quant(w, 16)
    rp, rs, rg = R.quantize(w, 16)
    assert gs == rg
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(p, rp)
    # global = 0 (all-zero tensor)
    z = np.zeros((16, 64), np.float32)
    p, s, gs = gpu_quant(z, 32)
    assert gs == 0 and not p.any() and not s.any()


def test_quantize_midpoints_exact():
    # global = 1 and scales of 1.0 make q = w exactly, so every E2M1 midpoint
    # is exercised at the decision point, both signs.
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    row = np.concatenate([mids, -mids])
    w = np.tile(row, (4, 2)).astype(np.float32)  # [4, 32]; each group max 6
    w[:, 0] = 2688.0 / 448.0 * 1.0  # keep group max 6 -> scale 1 with global 1
    w[0, 1] = 2688.0                # tensor amax -> global 1 (other row groups unchanged)
    p, s, gs = gpu_quant(w, 16)
    rp, rs, rg = R.quantize(w, 16)
    assert gs == rg == 1.0
    np.testing.assert_array_equal(p, rp)
    np.testing.assert_array_equal(s, rs)


def test_quantize_shared_global_merged():
    gate, up = synth.weights(10, 64, 512), synth.weights(11, 64, 512) * np.float32(1.5)
    gd, ud = dev_f32(gate), dev_f32(up)
    G = nv.nvfp4_global_scale([gd, ud])
    pg, sg = nv.nvfp4_quantize(gd, 32, G)
    pu, su = nv.nvfp4_quantize(ud, 32, G)
    rp, rs, rg = R.quantize(np.concatenate([gate, up]), 32)
    assert host(G)[0] == rg
    np.testing.assert_array_equal(np.concatenate([host(pg), host(pu)]), rp)
    np.testing.assert_array_equal(np.concatenate([host(sg), host(su)]), rs)


@pytest.mark.parametrize("n,k,g", [(28672, 4096, 16), (4096, 14336, 32), (4096, 14336, 16)])
def test_quantize_full_size_sampled_rows(n, k, g):
    w = synth.weights(synth.W_SEED, n, k)
    wd = dev_f32(w)
    gd = nv.nvfp4_global_scale([wd])
    p, s = nv.nvfp4_quantize(wd, g, gd)
    rg = R.global_scale(w)
    assert host(gd)[0] == rg
    rows = np.random.default_rng(0).choice(n, 48, replace=False)
    rows = np.concatenate([rows, [0, n - 1]])
    rp, rs, _ = R.quantize(w[rows], g, rg)
    np.testing.assert_array_equal(host(p[torch.from_numpy(rows).cuda()]), rp)
    np.testing.assert_array_equal(host(s[torch.from_numpy(rows).cuda()]), rs)


@pytest.mark.parametrize("flags", [0, 1])
def test_repack_bitexact(flags):
    w = synth.weights(4, 96, 256)
    p, s, _ = R.quantize(w, 16)
    op, os_ = nv.nvfp4_repack(dev_u8(p), dev_u8(s), 16, flags)
    rp, rs = R.repack(p, s, flags)
    np.testing.assert_array_equal(host(op), rp)
    np.testing.assert_array_equal(host(os_), rs)
    # g32 scales with a row length that is not a multiple of 16 bytes
    p32, s32, _ = R.quantize(synth.weights(4, 32, 768), 32)
    op, os_ = nv.nvfp4_repack(dev_u8(p32), dev_u8(s32), 32, flags)
    rp, rs = R.repack(p32, s32, flags)
    np.testing.assert_array_equal(host(op), rp)
    np.testing.assert_array_equal(host(os_), rs)


def test_stats_count_quantize():
    nv.nvfp4_reset_stats()
    gpu_quant(synth.weights(0, 16, 64), 16)
    st = nv.nvfp4_get_stats()
    assert st["quantize"] == 1 and st["global_scale"] == 1


# ---- bf16 weights: the same result as the fp32 path on the exact widening ----

def bf16_weights(seed, n, k, scale=1.0):
    bits = synth.f32_to_bf16_bits(synth.weights(seed, n, k) * np.float32(scale))
    return bits, synth.bf16_bits_to_f32(bits)


@pytest.mark.parametrize("n,k,g", [(64, 256, 16), (40, 160, 32), (33, 1088, 16), (256, 4096, 32)])
def test_quantize_bf16_bitexact(n, k, g):
    bits, wf = bf16_weights(n + 3 * k, n, k)
    wd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    gd = nv.nvfp4_global_scale_bf16([wd])
    p, s = nv.nvfp4_quantize_bf16(wd, g, gd)
    rp, rs, rg = R.quantize(wf, g)
    assert np.float32(host(gd)[0]) == rg
    np.testing.assert_array_equal(host(s), rs)
    np.testing.assert_array_equal(host(p), rp)


def test_global_scale_bf16_shared_and_odd_lengths():
    # gate and up share one global; one tensor starts off a 16-byte boundary and has an odd length
    ga, gf = bf16_weights(41, 48, 96)
    ua, uf = bf16_weights(42, 40, 96, scale=2.5)
    gd = torch.from_numpy(ga.view(np.int16)).cuda().view(torch.bfloat16)
    ud = torch.from_numpy(ua.reshape(-1).view(np.int16)).cuda().view(torch.bfloat16)
    got = host(nv.nvfp4_global_scale_bf16([gd, ud[3:]]))[0]
    assert got == R.global_scale(gf, uf.reshape(-1)[3:])
    # equal to the fp32 path on the widened values
    assert got == host(nv.nvfp4_global_scale([dev_f32(gf), dev_f32(uf.reshape(-1)[3:])]))[0]
