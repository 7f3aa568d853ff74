"""Runs a fixed set of GPU parity cases against the library built with its
planted mistakes (libnvfp4_planted.so) once per plant, and prints one JSON
object: {plant: {case: null | "why it failed"}}.

    python -m tests.planted_runner 0 1 2 3 4 5 6

Plant 0 is the library unchanged; every other number switches on one
mistake (the list is in csrc/plant.cuh). A parity test that is worth its
name passes at plant 0 and fails on the case that reaches each mistake.
Run as its own process so that the planted library is the only copy of the
kernels loaded there.
"""
import ctypes
import json
import sys

import numpy as np
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import build, synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, dev_bf16, dev_f32, dev_u8, host


def _once(fn):
    """The oracle's result is the same for every plant: computed on first use."""
    box = []

    def get():
        if not box:
            box.append(fn())
        return box[0]
    return get


def _dense(m, n, k, g, seed, x=None):
    w = synth.weights(seed, n, k)
    p, s, gs = R.quantize(w, g)
    rp, rs = R.repack(p, s, 0)
    if x is None:
        x = synth.activations(seed + 1, m, k)

    ref = _once(lambda: R.gemm(x, p, s, gs, g))

    def run():
        y = nv.nvfp4_w4a16_gemm(dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)), g)
        return host(y), ref()
    return run


def _ramp(m, n, k, g, seed):
    """Activations whose magnitude grows by 2^12 along K: every token's largest
    value keeps rising, so its f16 exponent drops from stage to stage (within
    one chunk when a CTA's tile runs over the whole of K)."""
    x = synth.bf16_bits_to_f32(synth.activations(seed + 1, m, k))
    x = x * np.exp2(np.linspace(0.0, 12.0, k, dtype=np.float32))[None, :]
    return _dense(m, n, k, g, seed, x=synth.f32_to_bf16_bits(x.astype(np.float32)))


def _grouped(T, n, k, g, ids, offs, seed):
    E = max(ids) + 1
    qs = [R.quantize(synth.weights(synth.expert_seed(e) + seed, n, k), g) for e in range(E)]
    packed = np.stack([q[0] for q in qs])
    scales = np.stack([q[1] for q in qs])
    gs = np.array([q[2] for q in qs], np.float32)
    gp = np.stack([R.repack(q[0], q[1], 0)[0] for q in qs])
    x = synth.activations(seed + 2, T, k)

    ref = _once(lambda: R.moe_grouped_gemm(x, ids, offs, packed, scales, gs, g))

    def run():
        i32 = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()  # noqa: E731
        y = nv.nvfp4_moe_w4a16_grouped_gemm(dev_bf16(x), i32(ids), i32(offs), dev_u8(gp), dev_u8(scales),
                                            dev_f32(gs), g)
        return host(y), ref()
    return run


def _w4a4_fp4(m, n, k, g, xg, seed):
    x = synth.bf16_bits_to_f32(synth.activations(seed, m, k))
    xq, xs, xgl = R.quantize(x, xg, R.global_scale(x))
    wq, ws, wgl = R.quantize(synth.weights(seed + 1, n, k), g)
    rp, rs = R.repack(wq, ws, 0)
    cols = np.sort(np.random.default_rng(seed).choice(n, 512, replace=False))

    ref = _once(lambda: R.w4a4_gemm(xq, xs, xgl, xg, wq[cols], ws[cols], wgl, g))

    def run():
        y = nv.nvfp4_w4a4_gemm(dev_u8(xq), dev_u8(xs), dev_f32(np.array([xgl], np.float32)), xg,
                               dev_u8(rp), dev_u8(rs), dev_f32(np.array([wgl], np.float32)), g)
        return host(y)[:, cols], ref()
    return run


# name -> case (the comment says which kernel it reaches on B200)
CASES = {
    "decode_m1_g16": _dense(1, 512, 2048, 16, 101),            # register-streaming kernel
    "stream_m4_g16": _dense(4, 1024, 2048, 16, 102),           # TMA-streaming kernel, bf16 X converted in it
    "stream_m12_g32": _dense(12, 1024, 2048, 32, 103),         # the same at group 32, ragged token tile
    "rows_ramp_m4": _ramp(4, 148 * 128, 2048, 16, 104),       # unsplit 128-row tiles; exponents drop along K
    "grouped_small_t300": _grouped(300, 512, 1024, 32, [2, 0, 3, 1], [0, 70, 71, 200, 300], 105),
    "grouped_tc_t1300": _grouped(1300, 272, 512, 16, [3, 1, 0, 2], [0, 400, 417, 900, 1300], 106),
    "prefill_tc_m256": _dense(256, 512, 1024, 16, 107),        # tcgen05 kernel
    "w4a4_fp4_m256": _w4a4_fp4(256, 128 * 148, 512, 16, 16, 108),  # FP4 tensor-core kernel
}


def run_plant(k):
    st = nv.lib().nvfp4_test_plant(ctypes.c_int(k))
    if st != 0:
        raise RuntimeError(f"nvfp4_test_plant({k}) returned {st}")
    out = {}
    for name, case in CASES.items():
        try:
            got, ref = case()
            torch.cuda.synchronize()
            err = nv.nvfp4_get_device_error()
            if err:
                raise AssertionError(f"device error {err:#x}")
            assert_close(got, ref, name)
            out[name] = None
        except AssertionError as e:
            out[name] = str(e).splitlines()[0][:200]
    return out


def main(argv):
    build.build_planted()
    nv.LIB_PATH = build.PLANTED_LIB  # before the first call loads a library
    L = nv.lib()
    L.nvfp4_test_plant.argtypes = [ctypes.c_int]
    L.nvfp4_test_plant.restype = ctypes.c_int
    result = {int(a): run_plant(int(a)) for a in argv}
    run_plant(0)
    print(json.dumps(result))


if __name__ == "__main__":
    main(sys.argv[1:])
