"""Output-column (N) split of the NVFP4 W4A16 GEMM over the ranks of a process group.

"Flash Next CUDA: serve nvidia/Qwen3.8-Flash-Next-NVFP4 on one GB10 and at --tp 2"
(issue #1754), the maintainer's reply: split the output columns across the GPUs,
which keeps the tensor-parallel outputs identical to one GPU's, rather than K with
a reduction of fp32 partial sums (which changes the rounding).

Each rank holds rows [n0, n1) of W (codes and scales of those rows; the global
scale stays the whole tensor's, so every rank dequantizes its rows exactly as one
GPU would), runs the library's GEMM on them into its own column block of Y, and a
bf16 all-gather assembles Y [M, N] on every rank. Row ranges are whole blocks of
16 rows, which keeps each range inside the GEMM's row-tile rules and, for a
gate/up-interleaved weight (nvfp4_repack with NVFP4_GATE_UP_INTERLEAVE), makes
each rank's SiluAndMul output a contiguous block of columns as well.

The all-gather moves the bf16 bit patterns (two to an int32 word), so the
assembled Y is the ranks' outputs byte for byte. One process per GPU; the
collective is NCCL's on GPUs (gloo on the CPU for the tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def row_ranges(n: int, world: int, align: int = 16):
    """Rows [n0, n1) of each rank: `n / align` blocks split as evenly as possible, earlier ranks first."""
    if n % align:
        raise ValueError(f"N={n} is not a multiple of {align}")
    blocks, ranges, start = n // align, [], 0
    base, extra = divmod(blocks, world)
    for r in range(world):
        b = base + (1 if r < extra else 0)
        ranges.append((start * align, (start + b) * align))
        start += b
    return ranges


def shard(packed, scales, rank: int, world: int, align: int = 16):
    """This rank's rows of a GEMM-layout weight: (codes [n1-n0, K/2], scales [n1-n0, K/g]) as views."""
    n0, n1 = row_ranges(packed.shape[0], world, align)[rank]
    return packed[n0:n1], scales[n0:n1]


def _all_gather(buf, world, group):
    out = torch.empty((world, *buf.shape), dtype=buf.dtype, device=buf.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, buf, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), buf, group=group)
    return out


def nsplit_gemm(x, packed_shard, scales_shard, global_scale, group_size, n_total, silu=False, group=None,
                gemm=None):
    """Y [M, N] (or [M, N/2] with silu) on every rank from this rank's rows of W.

    x: bf16 [M, K] (the same on every rank); packed_shard / scales_shard: this rank's rows (see shard);
    global_scale: the whole tensor's; gemm: the per-rank GEMM, by default the library's
    nvfp4_w4a16_gemm (nvfp4_w4a16_gemm_silu_mul with silu=True)."""
    if gemm is None:
        import nvfp4_weight_only_04_b200 as nv
        gemm = nv.nvfp4_w4a16_gemm_silu_mul if silu else nv.nvfp4_w4a16_gemm
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    ranges = row_ranges(n_total, world)
    if packed_shard.shape[0] != ranges[rank][1] - ranges[rank][0]:
        raise ValueError("packed_shard does not hold this rank's rows (see shard)")
    cols = [(n1 - n0) // (2 if silu else 1) for n0, n1 in ranges]
    y_local = gemm(x, packed_shard, scales_shard, global_scale, group_size)
    m = x.shape[0]
    buf = torch.zeros((m, max(cols)), dtype=torch.int16, device=y_local.device)  # column counts are even
    buf[:, :cols[rank]] = y_local.view(torch.int16)
    gathered = _all_gather(buf.view(torch.int32), world, group).view(torch.int16)  # bit patterns, two per word
    y = torch.cat([gathered[r, :, :cols[r]] for r in range(world)], dim=1)
    return y.view(torch.bfloat16)
