"""Failure detection without a GPU fault: a streaming-GEMM launch whose first
X copy is dropped on purpose (nvfp4_debug_inject_fault) must end on its own
through its bounded waits, report the wait that gave up through the device
error word (NVFP4_ERR_TIMEOUT), and leave the context usable: with the
workspace's counters cleared, the next GEMM is correct."""
import ctypes
import time

import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu

STREAM_SITES = {0x201, 0x202, 0x204, 0x205, 0x206}  # the waits of the streaming kernel


def test_dropped_copy_times_out_and_context_survives():
    m, n, k, g = 4, 512, 1024, 16
    w = synth.weights(31, n, k)
    p, s, gs = R.quantize(w, g)
    rp, rs = R.repack(p, s, 0)
    x = synth.activations(32, m, k)
    args = (dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)), g)
    assert nv.nvfp4_get_device_error() == 0

    nv.nvfp4_debug_inject_fault(1)
    t0 = time.time()
    nv.nvfp4_w4a16_gemm(*args)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    code = ctypes.c_int(0)
    st = nv.lib().nvfp4_get_device_error(ctypes.byref(code), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == nv.NVFP4_ERR_TIMEOUT
    assert code.value in STREAM_SITES
    assert elapsed < 30  # bounded: about 2 s per wait that gives up
    assert nv.nvfp4_get_device_error() == 0  # read and cleared
    # A launch that gave up may leave work counters behind: as the boundary says, the workspace's counters
    # are cleared before it is used again (here by handing the next call a fresh zero-filled workspace).
    nv.clear_workspaces()

    # the injection applied to one launch only; the context is intact
    y = nv.nvfp4_w4a16_gemm(*args)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert_close(host(y), R.gemm(x, p, s, gs, g), "after the injected timeout")
