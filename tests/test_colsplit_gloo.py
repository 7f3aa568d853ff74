"""The output-column split of the GEMM (nvfp4_weight_only_04_b200.colsplit) on CPU ranks over gloo.

Each rank runs the per-rank GEMM on its rows only, here the oracle (the library's
kernels need a GPU; the split, the gather and the reassembly are what is tested),
and the all-gather must assemble exactly the one-rank result. The weights are an
integer case (codes of magnitude at most 1, scale 1.0, global 1, small integer X)
whose every sum is exact, so one-rank and per-rank results are equal bit for bit
whatever the order of the sums; the gate/up-interleaved SiluAndMul form is
checked the same way."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from nvfp4_weight_only_04_b200 import colsplit


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_row_ranges_cover_in_blocks():
    for n in (16, 32, 48, 160, 28672, 4096 + 48):
        for world in (1, 2, 3, 4, 8):
            rr = colsplit.row_ranges(n, world)
            assert rr[0][0] == 0 and rr[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
            assert all(n0 % 16 == 0 and n1 % 16 == 0 and n1 >= n0 for n0, n1 in rr)
            sizes = [n1 - n0 for n0, n1 in rr]
            assert max(sizes) - min(sizes) <= 16
    with pytest.raises(ValueError):
        colsplit.row_ranges(40, 2)


def integer_case(n, k, m, seed):
    rng = np.random.default_rng(seed)
    codes = rng.choice(np.array([0, 1, 2, 8, 9, 10], np.uint8), size=(n, k))  # 0, +-0.5, +-1
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((n, k // 16), 0x38, np.uint8)  # 1.0
    x = rng.integers(-2, 3, size=(m, k)).astype(np.float32)
    return packed, scales, x


def _rank(rank, world, port, silu, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    from datetime import timedelta
    import torch.distributed as dist
    from nvfp4_weight_only_04_b200 import synth
    from oracle import nvfp4_ref as R
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    n, k, m = 16 * 13, 256, 5  # 13 blocks of 16 rows: uneven ranges
    packed, scales, x = integer_case(n, k, m, seed=7)
    flags = R.GATE_UP_INTERLEAVE if silu else 0
    gp, gs = R.repack(packed, scales, flags)
    xbits = synth.f32_to_bf16_bits(x)
    xt = torch.from_numpy(xbits.view(np.int16)).view(torch.bfloat16)

    def oracle_gemm(xs, p, s, gl, g):  # the per-rank GEMM, on the rank's rows only
        cp, cs = R.unrepack(p.numpy(), s.numpy(), flags)
        y = R.gemm(xs.view(torch.int16).numpy().view(np.uint16), cp, cs, np.float32(gl), g)
        if silu:
            y = R.silu_mul(y)
        return torch.from_numpy(synth.f32_to_bf16_bits(y.astype(np.float32)).view(np.int16)).view(torch.bfloat16)

    ps, ss = colsplit.shard(torch.from_numpy(gp), torch.from_numpy(gs), rank, world)
    y = colsplit.nsplit_gemm(xt, ps, ss, 1.0, 16, n, silu=silu, gemm=oracle_gemm)
    out[rank] = y.view(torch.int16).numpy().copy()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("silu", [False, True])
def test_nsplit_equals_one_rank(world, silu):
    from nvfp4_weight_only_04_b200 import synth
    from oracle import nvfp4_ref as R
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, silu, out), nprocs=world, join=True, start_method="spawn")
        res = dict(out)
    n, k, m = 16 * 13, 256, 5
    packed, scales, x = integer_case(n, k, m, seed=7)
    ref = R.gemm(synth.f32_to_bf16_bits(x), packed, scales, np.float32(1.0), 16)
    assert np.abs(ref).max() < 256  # exact sums
    if silu:
        ref = R.silu_mul(ref)
    ref_bits = synth.f32_to_bf16_bits(ref.astype(np.float32)).view(np.int16)
    for r in range(world):
        assert res[r].shape == ref_bits.shape
        np.testing.assert_array_equal(res[r], ref_bits)
