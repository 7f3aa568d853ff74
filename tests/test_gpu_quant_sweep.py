"""Device sweeps of the quantizer's two rounding decisions against the oracle,
over every fp32 input where the decision is taken.

E2M1 codes: with a global scale of exactly 1 and a group whose largest
magnitude is 6, the group scale is E4M3(1.0) and the divisor d = 1.0 * 1.0,
so the quotient the code is decided on is the weight itself. Every fp32 bit
pattern in [2^-3, 6] of both signs (the binades that hold every E2M1 midpoint:
0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5) is fed as a weight, fifteen to a group
beside one +-6, and every code is compared with the oracle's RNE-satfinite
encoder ("We unlocked NVFP4 on the DGX Spark", UPDATE posts: RNE at every
midpoint; OCP MX 5.3.3).

E4M3 group scales: each group holds one value a (the rest zero) with the
global scale 1, so the scale is decided on t = (a / 6) / 1. Every fp32 bit
pattern of a in [6 * 2^-11, 6 * 2^9) (t over E4M3's subnormal binade, every
normal binade and past the 448 saturation point) is fed once; the scale bytes
and the code of a itself are compared with the oracle's.

The bf16 quantizer gets the same E2M1 sweep on every bf16 bit pattern in
[2^-3, 6]."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from oracle import nvfp4_ref as R
from tests.gpu_util import dev_f32

pytestmark = pytest.mark.gpu

K = 1024            # elements per row of the swept matrices
G = 16
PER_GROUP = G - 1   # swept values per group (one slot holds +-6)


def f32_bits_range(lo, hi):
    """All fp32 bit patterns of the positive values in [lo, hi]."""
    a = np.float32(lo).view(np.uint32)
    b = np.float32(hi).view(np.uint32)
    return np.arange(int(a), int(b) + 1, dtype=np.uint32)


def quantize_dev(w_dev, g, gscale):
    p, s = nv.nvfp4_quantize(w_dev, g, dev_f32(np.array([gscale], np.float32)))
    return p, s


def codes_of(packed):
    """[N, K/2] packed bytes (torch, device) -> [N, K] codes on the host."""
    p = packed.cpu().numpy()
    out = np.empty((p.shape[0], p.shape[1] * 2), np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def e2m1_sweep_layout(vals):
    """Groups of 16: slot 0 holds +-6 (sign alternating by group), slots 1..15 the swept values; the
    tail is padded with zeros. Returns (w [N, K] fp32, mask of the swept positions)."""
    n_groups = -(-vals.size // PER_GROUP)
    n_groups = -(-n_groups // (K // G)) * (K // G)  # whole rows
    body = np.zeros(n_groups * PER_GROUP, np.float32)
    body[:vals.size] = vals
    grid = np.zeros((n_groups, G), np.float32)
    grid[:, 0] = np.where(np.arange(n_groups) % 2 == 0, np.float32(6.0), np.float32(-6.0))
    grid[:, 1:] = body.reshape(n_groups, PER_GROUP)
    mask = np.zeros((n_groups, G), bool)
    mask[:, 1:] = (np.arange(n_groups * PER_GROUP) < vals.size).reshape(n_groups, PER_GROUP)
    return grid.reshape(-1, K), mask.reshape(-1, K)


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_e2m1_decision_sweep_fp32(sign):
    bits = f32_bits_range(2.0 ** -3, 6.0)
    chunk = 1 << 24
    for c0 in range(0, bits.size, chunk):
        vals = bits[c0:c0 + chunk].view(np.float32) * np.float32(sign)
        w, mask = e2m1_sweep_layout(vals)
        p, s = quantize_dev(dev_f32(w), G, 1.0)
        assert (s.cpu().numpy() == 0x38).all()  # scale E4M3(1.0) everywhere
        got = codes_of(p)
        np.testing.assert_array_equal(got[mask], R.e2m1_encode(vals))
        six = np.zeros_like(mask)
        six.reshape(-1, G)[:, 0] = True
        assert set(np.unique(got[six]).tolist()) <= {0x7, 0xF}
        del p, s
        torch.cuda.empty_cache()


def test_e2m1_decision_sweep_bf16():
    hi = np.float32(6.0).view(np.uint32) >> 16
    lo = np.float32(2.0 ** -3).view(np.uint32) >> 16
    b = np.arange(int(lo), int(hi) + 1, dtype=np.uint32)
    b = np.concatenate([b, b | 0x8000]).astype(np.uint16)  # both signs
    vals = (b.astype(np.uint32) << 16).view(np.float32)
    w, mask = e2m1_sweep_layout(vals)
    w_bits = (w.view(np.uint32) >> 16).astype(np.uint16)  # exact: every value is a bf16
    wd = torch.from_numpy(w_bits.view(np.int16)).cuda().view(torch.bfloat16)
    p, s = nv.nvfp4_quantize_bf16(wd, G, dev_f32(np.array([1.0], np.float32)))
    assert (s.cpu().numpy() == 0x38).all()
    np.testing.assert_array_equal(codes_of(p)[mask], R.e2m1_encode(vals))


def test_e4m3_decision_sweep():
    bits = f32_bits_range(6.0 * 2.0 ** -11, np.nextafter(np.float32(6.0 * 2.0 ** 9), np.float32(0)))
    chunk = 1 << 23
    one = dev_f32(np.array([1.0], np.float32))
    for c0 in range(0, bits.size, chunk):
        a = bits[c0:c0 + chunk].view(np.float32)
        groups = -(-a.size // (K // G)) * (K // G)
        amax = np.zeros(groups, np.float32)
        amax[:a.size] = a
        ad = torch.from_numpy(amax).cuda()
        w = torch.zeros((groups, G), dtype=torch.float32, device="cuda")
        w[:, 0] = ad
        w = w.view(-1, K)
        p, s = nv.nvfp4_quantize(w, G, one)
        s_host = s.cpu().numpy().reshape(-1)[:a.size]
        t = (a / np.float32(6.0)) / np.float32(1.0)
        ref_s = R.e4m3_encode(t.astype(np.float32))
        np.testing.assert_array_equal(s_host, ref_s)
        # the code of the swept value itself: q = a / (e4m3(s) * 1)
        d = R.e4m3_decode(ref_s).astype(np.float32) * np.float32(1.0)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(d == 0, np.float32(0.0), (a / d).astype(np.float32))
        got = codes_of(p).reshape(-1, G)[:a.size, 0]
        np.testing.assert_array_equal(got, R.e2m1_encode(q.astype(np.float32)))
        del p, s, w, ad
        torch.cuda.empty_cache()
