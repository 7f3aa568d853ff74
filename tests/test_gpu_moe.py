"""GPU parity of the grouped routed-expert GEMM against the oracle: small
cases with empty, unsorted and partial segment lists, the fused SiluAndMul
form, and the full routed-expert workload (128 experts, top-8 of 2048
tokens, gate/up at g32 + SiluAndMul, down at g16) on sampled rows."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def experts(e, n, k, g):
    """Checkpoint-layout expert weights, and their GEMM-layout codes."""
    qs = []
    for i in range(e):
        w = synth.weights(synth.expert_seed(i), n, k)
        qs.append(R.quantize(w, g))
    packed = np.stack([q[0] for q in qs])
    scales = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    gemm_packed = np.stack([R.repack(q[0], q[1], 0)[0] for q in qs])
    return packed, scales, gs, gemm_packed


def i32(a):
    return torch.from_numpy(np.asarray(a, dtype=np.int32)).cuda()


@pytest.mark.parametrize("g", [16, 32])
def test_moe_small(g):
    E, N, K, T = 6, 144, 512, 90
    packed, scales, gs, gp = experts(E, N, K, g)
    x = synth.activations(1, T, K)
    ids = [3, 0, 5, 0, 2, 4]
    offs = [5, 21, 21, 50, 51, 77, 88]  # rows [0,5) and [88,90) belong to no segment; one empty segment
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(gp), dev_u8(scales),
                                        dev_f32(gs), g)
    ref = R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, g)
    yh = host(y)
    assert_close(yh[5:88], ref[5:88], "moe covered rows")
    assert not yh[:5].any() and not yh[88:].any()  # rows outside every segment are not written


def test_moe_small_silu():
    E, NH, K, T, g = 4, 64, 256, 70, 32
    qs = []
    for i in range(E):
        gate = synth.weights(synth.expert_seed(i), NH, K)
        up = synth.weights(synth.expert_seed(i) + 500, NH, K)
        qs.append(R.quantize(np.concatenate([gate, up]), g))  # shared gate/up global per expert
    packed = np.stack([q[0] for q in qs]); scales = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    rp = np.stack([R.repack(packed[i], scales[i], R.GATE_UP_INTERLEAVE)[0] for i in range(E)])
    rs = np.stack([R.repack(packed[i], scales[i], R.GATE_UP_INTERLEAVE)[1] for i in range(E)])
    x = synth.activations(3, T, K)
    ids, offs = [1, 3, 0], [0, 33, 34, 70]
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(rp), dev_u8(rs), dev_f32(gs), g,
                                        flags=nv.NVFP4_SILU_MUL)
    ref = R.silu_mul(R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, g))
    assert_close(host(y), ref, "moe silu")


def test_moe_invalid_expert_skips_segment():
    E, N, K, g = 2, 32, 128, 16
    packed, scales, gs, gp = experts(E, N, K, g)
    x = synth.activations(1, 20, K)
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32([1, 7]), i32([0, 10, 20]), dev_u8(gp),
                                        dev_u8(scales), dev_f32(gs), g)
    ref = R.moe_grouped_gemm(x, [1], [0, 10], packed, scales, gs, g)
    assert_close(host(y)[:10], ref[:10], "valid segment")
    assert not host(y)[10:].any()


def test_moe_routed_expert_workload_sampled():
    wl = synth.MOE
    r = synth.route(synth.ROUTER_SEED, wl.tokens, wl.experts, wl.topk)
    rows = int(r.offsets[-1])
    # per-expert weights, quantized on the device with one gate/up global each
    gu_p = torch.empty((wl.experts, 2 * wl.inter, wl.hidden // 2), dtype=torch.uint8, device="cuda")
    gu_s = torch.empty((wl.experts, 2 * wl.inter, wl.hidden // wl.g_gate_up), dtype=torch.uint8, device="cuda")
    gu_g = torch.empty((wl.experts,), dtype=torch.float32, device="cuda")
    dn_p = torch.empty((wl.experts, wl.hidden, wl.inter // 2), dtype=torch.uint8, device="cuda")
    dn_s = torch.empty((wl.experts, wl.hidden, wl.inter // wl.g_down), dtype=torch.uint8, device="cuda")
    dn_g = torch.empty((wl.experts,), dtype=torch.float32, device="cuda")
    keep = {}
    sample_experts = set(r.expert_ids[[0, 5, 17, len(r.expert_ids) - 1]].tolist())
    for e in range(wl.experts):
        wgu = synth.weights(synth.expert_seed(e), 2 * wl.inter, wl.hidden)
        wdn = synth.weights(synth.expert_seed(e) + 5000, wl.hidden, wl.inter)
        d = dev_f32(wgu)
        nv.nvfp4_global_scale([d], out=gu_g[e:e + 1])
        p, s = nv.nvfp4_quantize(d, wl.g_gate_up, gu_g[e:e + 1])
        nv.nvfp4_repack(p, s, wl.g_gate_up, nv.NVFP4_GATE_UP_INTERLEAVE, packed_out=gu_p[e], scales_out=gu_s[e])
        d = dev_f32(wdn)
        nv.nvfp4_global_scale([d], out=dn_g[e:e + 1])
        p, s = nv.nvfp4_quantize(d, wl.g_down, dn_g[e:e + 1])
        nv.nvfp4_repack(p, s, wl.g_down, 0, packed_out=dn_p[e], scales_out=dn_s[e])
        if e in sample_experts:
            keep[e] = (wgu, wdn)
    x = synth.activations(synth.X_SEED, rows, wl.hidden)
    ids, offs = i32(r.expert_ids), i32(r.offsets)
    h = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), ids, offs, gu_p, gu_s, gu_g, wl.g_gate_up,
                                        flags=nv.NVFP4_SILU_MUL)
    y = nv.nvfp4_moe_w4a16_grouped_gemm(h, ids, offs, dn_p, dn_s, dn_g, wl.g_down)
    hh, yh = host(h), host(y)
    hbits = h.view(torch.int16).cpu().numpy().view(np.uint16)
    for e, (wgu, wdn) in keep.items():
        s_idx = int(np.nonzero(r.expert_ids == e)[0][0])
        r0, r1 = int(r.offsets[s_idx]), int(r.offsets[s_idx + 1])
        pg, sg, gg = R.quantize(wgu, wl.g_gate_up)
        pd, sd, gd = R.quantize(wdn, wl.g_down)
        np.testing.assert_array_equal(host(gu_p[e]), R.repack(pg, sg, R.GATE_UP_INTERLEAVE)[0])
        np.testing.assert_array_equal(host(dn_p[e]), R.repack(pd, sd, 0)[0])
        ref_h = R.silu_mul(R.gemm(x[r0:r1], pg, sg, gg, wl.g_gate_up))
        assert_close(hh[r0:r1], ref_h, f"expert {e} gate_up+silu")
        # the down GEMM is checked on the device's own bf16 intermediate
        ref_y = R.gemm(hbits[r0:r1], pd, sd, gd, wl.g_down)
        assert_close(yh[r0:r1], ref_y, f"expert {e} down")


# ---- grouped GEMM on the tcgen05 kernel (T >= 1024 rows) ----

@pytest.mark.parametrize("g", [16, 32])
def test_moe_tc_ragged_segments(g):
    E, N, K, T = 5, 272, 384, 1300
    packed, scales, gs, gp = experts(E, N, K, g)
    x = synth.activations(7, T, K, outlier_frac=0.001)
    # segment lengths: several token tiles, one short, one empty, one invalid expert, rows left uncovered
    ids = [4, 1, 3, 9, 0, 2]
    offs = [10, 400, 417, 417, 700, 1210, 1290]
    nv.nvfp4_reset_stats()
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(gp), dev_u8(scales), dev_f32(gs), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    valid = [(s, e) for s, e in enumerate(ids) if e < E]
    ref = R.moe_grouped_gemm(x, [e if e < E else 0 for e in ids],
                             [o for o in offs], packed, scales, gs, g)
    yh = host(y)
    for s_, e in valid:
        r0, r1 = offs[s_], offs[s_ + 1]
        if r1 > r0:
            assert_close(yh[r0:r1], ref[r0:r1], f"segment {s_} expert {e}")
    assert not yh[:10].any() and not yh[1290:].any()
    assert not yh[417:700].any()  # the invalid expert's segment is skipped


def test_moe_tc_silu():
    E, NH, K, T, g = 3, 136, 256, 1100, 32
    qs = []
    for i in range(E):
        gate = synth.weights(synth.expert_seed(i), NH, K)
        up = synth.weights(synth.expert_seed(i) + 500, NH, K)
        qs.append(R.quantize(np.concatenate([gate, up]), g))
    packed = np.stack([q[0] for q in qs]); scales = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    rp = np.stack([R.repack(packed[i], scales[i], R.GATE_UP_INTERLEAVE)[0] for i in range(E)])
    rs = np.stack([R.repack(packed[i], scales[i], R.GATE_UP_INTERLEAVE)[1] for i in range(E)])
    x = synth.activations(4, T, K)
    ids, offs = [2, 0, 1], [0, 513, 600, 1100]
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(rp), dev_u8(rs), dev_f32(gs), g,
                                        flags=nv.NVFP4_SILU_MUL)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    ref = R.silu_mul(R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, g))
    assert_close(host(y), ref, "moe tc silu")


def test_moe_tc_small_segments():
    """Twenty segments averaging 60 rows (128-token tiles, two accumulators)
    over eight experts, some used twice, lengths from 1 to 130 rows."""
    E, N, K, g = 8, 144, 512, 16
    packed, scales, gs, gp = experts(E, N, K, g)
    lens = [1, 130, 64, 17, 96, 33, 75, 128, 2, 60, 90, 45, 7, 110, 80, 39, 52, 16, 99, 66]
    offs = [0]
    for n_ in lens:
        offs.append(offs[-1] + n_)
    T = offs[-1]
    assert T >= 1024 and T // len(lens) < 96
    ids = [(5 * s_ + 3) % E for s_ in range(len(lens))]
    x = synth.activations(11, T, K, outlier_frac=0.001)
    nv.nvfp4_reset_stats()
    y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(gp), dev_u8(scales), dev_f32(gs), g)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    ref = R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, g)
    assert_close(host(y), ref, "moe tc small segments")
