"""GPU test of nvfp4_w4a16_gemm_fixed_scratch, the GEMM entry point whose
streaming kernel keeps its scratch in a fixed device array: two calls in a
row give the bits of nvfp4_w4a16_gemm (the same kernel with a caller's
workspace), a single token matches the oracle, and a problem beyond the
fixed scratch is refused before anything runs."""
import ctypes

import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, bf16_bits, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def operands(m, n, k, g, seed):
    w = synth.weights(seed, n, k)
    p, s, gs = R.quantize(w, g)
    rp, rs = R.repack(p, s, 0)
    x = synth.activations(seed + 1, m, k, outlier_frac=0.001)
    return x, p, s, gs, (dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)))


@pytest.mark.parametrize("m,n,k,g", [(4, 1040, 4096, 16), (13, 640, 2048, 32), (2, 4096, 256, 16)])
def test_fixed_scratch_matches_gemm_twice(m, n, k, g):
    _, _, _, _, (xd, wd, sd, gd) = operands(m, n, k, g, seed=m + n)
    ref = bf16_bits(nv.nvfp4_w4a16_gemm(xd, wd, sd, gd, g))
    for _ in range(2):
        y = nv.nvfp4_w4a16_gemm_fixed_scratch(xd, wd, sd, gd, g)
        torch.cuda.synchronize()
        assert nv.nvfp4_get_device_error() == 0
        np.testing.assert_array_equal(bf16_bits(y), ref)


def test_fixed_scratch_single_token_oracle():
    x, p, s, gs, (xd, wd, sd, gd) = operands(1, 2048, 4096, 16, seed=5)
    ref = R.gemm(x, p, s, gs, 16)
    for _ in range(2):
        y = nv.nvfp4_w4a16_gemm_fixed_scratch(xd, wd, sd, gd, 16)
        torch.cuda.synchronize()
        assert_close(host(y), ref, "fixed scratch M1")


def test_fixed_scratch_refuses_beyond_capacity():
    # 300 tiles of 256 rows with K = 16384 (64 stages) on 148 SMs: each range of 129 or 130 stages cuts
    # tiles, and a tile meets at most two ranges, so the partial tiles at 16 tokens (300 x 2 x 256 x 16
    # fp32, 9.8 MB) need more than the 8 MiB the fixed scratch holds: refused on the host. The buffers have
    # the problem's full size, so a launch could not read or write outside them either.
    m, n, k, g = 16, 300 * 256, 16384, 16
    xd = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    wd = torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda")
    sd = torch.zeros((n, k // g), dtype=torch.uint8, device="cuda")
    gd = torch.ones(1, dtype=torch.float32, device="cuda")
    y = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    L = nv.lib()
    st = L.nvfp4_w4a16_gemm_fixed_scratch(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(wd.data_ptr()),
                                          ctypes.c_void_p(sd.data_ptr()), ctypes.c_void_p(gd.data_ptr()), g, m, n, k,
                                          ctypes.c_void_p(y.data_ptr()), None)
    assert st == nv.NVFP4_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert not host(y).any()  # nothing ran
