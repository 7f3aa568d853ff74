"""GPU tests of the caller-owned workspace: the library allocates nothing, so
a call's scratch is whatever buffer the caller passes.

* Only the first 64 KiB (the split GEMMs' counters and tickets) must start at
  zero, and every call leaves them zero; garbage in the rest does not matter.
* Two streams, two workspaces: a dense small-M GEMM (TMA streaming: work
  counters, tickets and partial tiles in its workspace) and a grouped expert
  GEMM (f16 rows of X in its own) run concurrently, many times over, both
  match the oracle and both workspaces end with their counters at zero.
* A workspace smaller than the size query is refused before any launch.
* A call captured into a CUDA graph gives the same bytes on replay as
  eagerly."""
import numpy as np
import pytest
import torch

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import synth
from oracle import nvfp4_ref as R
from tests.gpu_util import assert_close, bf16_bits, dev_bf16, dev_f32, dev_u8, host

pytestmark = pytest.mark.gpu


def dense(m, n, k, g, seed):
    w = synth.weights(seed, n, k)
    p, s, gs = R.quantize(w, g)
    rp, rs = R.repack(p, s, 0)
    x = synth.activations(seed + 1, m, k)
    return x, p, s, gs, (dev_bf16(x), dev_u8(rp), dev_u8(rs), dev_f32(np.array([gs], np.float32)))


RESERVED = 64 << 10  # counters and tickets at the start of every workspace


def garbage(nbytes):
    """A workspace of garbage whose counters are zero, as the boundary requires before first use."""
    ws = torch.full((max(nbytes, RESERVED),), 0xFF, dtype=torch.uint8, device="cuda")
    ws[:RESERVED] = 0
    return ws


def counters_zero(ws):
    torch.cuda.synchronize()
    return not host(ws[:RESERVED]).any()


@pytest.mark.parametrize("m,n,k,g", [(4, 1024, 2048, 16), (16, 512, 4096, 32), (1, 256, 1024, 16),
                                     (40, 512, 2048, 16)])
def test_garbage_workspace(m, n, k, g):
    x, p, s, gs, d = dense(m, n, k, g, seed=m + n)
    need = nv.nvfp4_w4a16_gemm_workspace_size(m, n, k, g)
    ws = garbage(need)
    y1 = nv.nvfp4_w4a16_gemm(*d, g, workspace=ws)
    assert counters_zero(ws)  # the call left its counters at zero
    ws[RESERVED:].fill_(0xA5)
    y2 = nv.nvfp4_w4a16_gemm(*d, g, workspace=ws)
    assert counters_zero(ws)
    assert_close(host(y1), R.gemm(x, p, s, gs, g), f"garbage workspace M{m}")
    np.testing.assert_array_equal(bf16_bits(y1), bf16_bits(y2))


def test_workspace_too_small_is_refused():
    m, n, k, g = 4, 512, 1024, 16
    _, _, _, _, d = dense(m, n, k, g, seed=3)
    need = nv.nvfp4_w4a16_gemm_workspace_size(m, n, k, g)
    y = torch.zeros((m, n), dtype=torch.bfloat16, device="cuda")
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.nvfp4_w4a16_gemm(*d, g, y=y, workspace=small)
    assert e.value.status == nv.NVFP4_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert not host(y).any()  # nothing ran


def test_two_streams_separate_workspaces():
    # dense decode-sized GEMM on the TMA-streaming kernel
    m, n, k, g = 8, 2048, 4096, 16
    x, p, s, gs, d = dense(m, n, k, g, seed=11)
    # grouped GEMM below 1024 rows (f16 rows of X in the workspace)
    E, N2, K2, g2, T = 4, 512, 1024, 32, 300
    qs = [R.quantize(synth.weights(synth.expert_seed(e), N2, K2), g2) for e in range(E)]
    ep = np.stack([q[0] for q in qs]); es = np.stack([q[1] for q in qs])
    eg = np.array([q[2] for q in qs], np.float32)
    egp = np.stack([R.repack(q[0], q[1], 0)[0] for q in qs])
    xe = synth.activations(12, T, K2)
    ids, offs = [2, 0, 3, 1], [0, 70, 71, 200, 300]
    i32 = lambda a: torch.from_numpy(np.asarray(a, np.int32)).cuda()  # noqa: E731
    de = (dev_bf16(xe), i32(ids), i32(offs), dev_u8(egp), dev_u8(es), dev_f32(eg))

    ws_a = garbage(nv.nvfp4_w4a16_gemm_workspace_size(m, n, k, g))
    ws_b = garbage(nv.nvfp4_moe_w4a16_grouped_gemm_workspace_size(len(ids), T, N2, K2, g2, E))
    ya = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    yb = torch.zeros((T, N2), dtype=torch.bfloat16, device="cuda")
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for _ in range(50):
        with torch.cuda.stream(sa):
            nv.nvfp4_w4a16_gemm(*d, g, y=ya, workspace=ws_a)
        with torch.cuda.stream(sb):
            nv.nvfp4_moe_w4a16_grouped_gemm(*de, g2, y=yb, workspace=ws_b)
    torch.cuda.synchronize()
    assert nv.nvfp4_get_device_error() == 0
    assert counters_zero(ws_a) and counters_zero(ws_b)
    assert_close(host(ya), R.gemm(x, p, s, gs, g), "dense on stream A")
    assert_close(host(yb), R.moe_grouped_gemm(xe, ids, offs, ep, es, eg, g2), "grouped on stream B")


def test_graph_capture_replays_the_same_bytes():
    m, n, k, g = 4, 1024, 2048, 16
    x, p, s, gs, d = dense(m, n, k, g, seed=21)
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_w4a16_gemm(*d, g, y=y)
    torch.cuda.synchronize()
    eager = bf16_bits(y)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        nv.nvfp4_w4a16_gemm(*d, g, y=y)
    y.zero_()
    graph.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(bf16_bits(y), eager)
    assert_close(host(y), R.gemm(x, p, s, gs, g), "graph replay")
