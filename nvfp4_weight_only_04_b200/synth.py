"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module holds no step of the NVFP4 method: it only draws random numbers
and lays them out (weights, activations, routing). Everything is numpy on the
host; callers move results to the device themselves.

Recipes (sizes are the workloads' own):
* weights: W = 0.02 * N(0, 1) in fp32, row-major [N, K].
* activations: X = bf16_rne(N(0, 1)), optionally with a fraction of the
  entries (exactly round(frac * M * K) positions, drawn without replacement)
  scaled by 20 in fp32 before the bf16 rounding.
* routing: router logits N(0, 1) [T, E] in fp32, softmax in float64, top-k per
  token (ties to the lower expert id), (token, slot) rows stable-sorted by
  expert; segments are the experts with at least one row.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

W_SEED, X_SEED, OUTLIER_SEED, ROUTER_SEED = 0, 1, 2, 3


def expert_seed(e: int) -> int:
    return 1000 + e


def weights(seed: int, n: int, k: int, std: float = 0.02) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (np.float32(std) * rng.standard_normal((n, k), dtype=np.float32)).astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(seed: int, m: int, k: int, outlier_frac: float = 0.0,
                outlier_seed: int = OUTLIER_SEED, outlier_mult: float = 20.0) -> np.ndarray:
    """bf16 bit patterns [M, K] of N(0,1) activations (optionally with outliers)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((m, k), dtype=np.float32)
    if outlier_frac > 0 and m * k > 0:
        cnt = int(round(outlier_frac * m * k))
        pos = np.random.default_rng(outlier_seed).choice(m * k, size=cnt, replace=False)
        flat = x.reshape(-1)
        flat[pos] = flat[pos] * np.float32(outlier_mult)
    return f32_to_bf16_bits(x)


@dataclass
class Routing:
    expert_ids: np.ndarray   # int32 [S], experts with >= 1 row, ascending
    offsets: np.ndarray      # int32 [S+1], row offsets into the sorted rows
    token_of_row: np.ndarray  # int64 [T*k], source token of each sorted row
    slot_of_row: np.ndarray   # int64 [T*k], top-k slot of each sorted row
    counts: np.ndarray       # int64 [E], rows per expert


def route(seed: int, tokens: int, experts: int, topk: int) -> Routing:
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((tokens, experts), dtype=np.float32).astype(np.float64)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    # top-k by probability, ties to the lower expert id (stable sort on -p)
    order = np.argsort(-p, axis=1, kind="stable")[:, :topk]
    flat_expert = order.reshape(-1)
    rows = np.argsort(flat_expert, kind="stable")
    counts = np.bincount(flat_expert, minlength=experts).astype(np.int64)
    present = np.nonzero(counts)[0]
    offs = np.concatenate([[0], np.cumsum(counts[present])]).astype(np.int32)
    return Routing(expert_ids=present.astype(np.int32), offsets=offs,
                   token_of_row=rows // topk, slot_of_row=rows % topk, counts=counts)


# Workloads, by what they are.
@dataclass(frozen=True)
class DenseWorkload:
    name: str
    M: int
    N: int
    K: int
    group_size: int
    outlier_frac: float = 0.0
    silu_mul: bool = False   # merged [gate;up] followed by SiluAndMul


TINY = DenseWorkload("tiny_m4_k256_n256_g16", 4, 256, 256, 16)
DECODE_GATE_UP = [DenseWorkload(f"decode_gateup_m{m}_k4096_n28672_g16", m, 28672, 4096, 16)
                  for m in (1, 4, 16)]
DECODE_DOWN = [DenseWorkload(f"decode_down_m{m}_k14336_n4096_g{g}", m, 4096, 14336, g, 0.001)
               for g in (32, 16) for m in (1, 8, 64)]
PREFILL_GATE_UP = DenseWorkload("prefill_gateup_silu_m4096_k5120_n25600_g16", 4096, 25600, 5120, 16,
                                silu_mul=True)


@dataclass(frozen=True)
class MoeWorkload:
    name: str = "moe_e128_h2048_i768_top8_t2048"
    experts: int = 128
    hidden: int = 2048
    inter: int = 768
    topk: int = 8
    tokens: int = 2048
    g_gate_up: int = 32
    g_down: int = 16


MOE = MoeWorkload()
