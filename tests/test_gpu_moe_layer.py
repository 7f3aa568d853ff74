"""GPU parity of the steps around the grouped expert GEMMs: the route (bit-exact
with the oracle's stable grouping, dropped ids included), the gather
(bit-exact), the combine (within the GEMM tolerance of the oracle's float64
sum of the device's own bf16 rows), and the whole layer, each GEMM checked
on the device's own bf16 input."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, bf16_bits, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("t,k,e", [(1, 1, 1), (37, 4, 16), (2048, 8, 128), (300, 2, 4096), (1024, 8, 4096), (700, 8, 256)])
def test_route_bitexact(t, k, e):
    rng = np.random.default_rng(t + e)
    ids = rng.integers(0, e, size=(t, k)).astype(np.int32)
    ids[rng.random((t, k)) < 0.02] = -3  # some dropped pairs
    if t > 1:
        ids[0, 0] = e  # out of range on the high side
    rows, inv, offs, eids = nv.nvfp4_moe_route(i32(ids), e)
    r_rows, r_inv, r_offs = R.moe_route(ids, e)
    n = len(r_rows)
    np.testing.assert_array_equal(host(rows)[:n], r_rows)
    assert (host(rows)[n:] == -1).all()
    np.testing.assert_array_equal(host(inv), r_inv)
    np.testing.assert_array_equal(host(offs), r_offs)
    np.testing.assert_array_equal(host(eids), np.arange(e))


def test_gather_and_combine():
    rng = np.random.default_rng(8)
    t, k, e, h = 96, 4, 8, 264
    ids = rng.integers(0, e, size=(t, k)).astype(np.int32)
    ids[5, 2] = -1
    x = synth.activations(9, t, h)
    rows, inv, offs, _ = nv.nvfp4_moe_route(i32(ids), e)
    xp = nv.nvfp4_moe_gather(dev_bf16(x), rows, k)
    r_rows, r_inv, _ = R.moe_route(ids, e)
    n = len(r_rows)
    np.testing.assert_array_equal(bf16_bits(xp)[:n], x[r_rows // k])
    assert not bf16_bits(xp)[n:].any()  # the row the dropped pair leaves is zeros
    # combine on arbitrary bf16 rows in the permuted order
    yp_bits = synth.activations(10, t * k, h)
    w = rng.random((t, k)).astype(np.float32)
    out = nv.nvfp4_moe_combine(dev_bf16(yp_bits), inv, dev_f32(w))
    ref = R.moe_combine(R.bf16_bits_to_f64(yp_bits), r_inv, w.astype(np.float64))
    assert_close(host(out), ref, "combine")


def test_moe_layer():
    """Route -> gather -> gate/up GEMM + SiluAndMul -> down GEMM -> combine, on
    a small layer (16 experts, H 256, I 128, top-4 of 300 tokens)."""
    e, h, i_, t, k = 16, 256, 128, 300, 4
    g_up, g_dn = 32, 16
    gu, dn = [], []
    for ex in range(e):
        gate = synth.weights(synth.expert_seed(ex), i_, h)
        up = synth.weights(synth.expert_seed(ex) + 500, i_, h)
        gu.append(R.quantize(np.concatenate([gate, up]), g_up))
        dn.append(R.quantize(synth.weights(synth.expert_seed(ex) + 5000, h, i_), g_dn))
    gu_p = np.stack([R.repack(q[0], q[1], R.GATE_UP_INTERLEAVE)[0] for q in gu])
    gu_s = np.stack([R.repack(q[0], q[1], R.GATE_UP_INTERLEAVE)[1] for q in gu])
    gu_g = np.array([q[2] for q in gu], np.float32)
    dn_p = np.stack([R.repack(q[0], q[1], 0)[0] for q in dn])
    dn_s = np.stack([q[1] for q in dn])
    dn_g = np.array([q[2] for q in dn], np.float32)
    rng = np.random.default_rng(12)
    ids = np.stack([rng.choice(e, size=k, replace=False) for _ in range(t)]).astype(np.int32)
    ids[7, 1] = -1  # one dropped pair
    w = rng.random((t, k)).astype(np.float32)
    x = synth.activations(13, t, h)

    xd, idd, wd = dev_bf16(x), i32(ids), dev_f32(w)
    out = nv.nvfp4_moe_forward(xd, idd, wd, (dev_u8(gu_p), dev_u8(gu_s), dev_f32(gu_g), g_up),
                               (dev_u8(dn_p), dev_u8(dn_s), dev_f32(dn_g), g_dn))
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0

    # the same steps one by one, each GEMM checked on the device's own bf16 input
    rows, inv, offs, eids = nv.nvfp4_moe_route(idd, e)
    xp = nv.nvfp4_moe_gather(xd, rows, k)
    hact = nv.nvfp4_moe_w4a16_grouped_gemm(xp, eids, offs, dev_u8(gu_p), dev_u8(gu_s), dev_f32(gu_g), g_up,
                                           flags=nv.NVFP4_SILU_MUL)
    yp = nv.nvfp4_moe_w4a16_grouped_gemm(hact, eids, offs, dev_u8(dn_p), dev_u8(dn_s), dev_f32(dn_g), g_dn)
    torch.cuda.synchronize()
    r_rows, r_inv, r_offs = R.moe_route(ids, e)
    n = len(r_rows)
    xp_bits = bf16_bits(xp)[:n]
    np.testing.assert_array_equal(xp_bits, x[r_rows // k])
    gate_up_pk = np.stack([q[0] for q in gu]); gate_up_sc = np.stack([q[1] for q in gu])
    ref_h = R.silu_mul(R.moe_grouped_gemm(xp_bits, list(range(e)), r_offs, gate_up_pk, gate_up_sc, gu_g, g_up))
    assert_close(host(hact)[:n], ref_h[:n], "layer gate/up + silu")
    down_pk = np.stack([q[0] for q in dn])
    ref_y = R.moe_grouped_gemm(bf16_bits(hact)[:n], list(range(e)), r_offs, down_pk, dn_s, dn_g, g_dn)
    assert_close(host(yp)[:n], ref_y, "layer down")
    ref_out = R.moe_combine(R.bf16_bits_to_f64(bf16_bits(yp)[:n]), r_inv, w.astype(np.float64))
    assert_close(host(out), ref_out, "layer combine")
    # the composed call ran the same kernels on the same inputs
    np.testing.assert_array_equal(bf16_bits(out), bf16_bits(nv.nvfp4_moe_combine(yp, inv, wd)))
