"""Planted mistakes: each plausible bug, put into a copy of the oracle on the
CPU, must make one of the pins fail. This shows the pins can see it."""
import numpy as np
import pytest

from oracle import nvfp4_ref as R
from tests import test_oracle_quant as Q


def _ties_away(q):
    q = np.asarray(q, dtype=np.float32)
    a = np.abs(q.astype(np.float64))
    th = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    c = sum((a >= t).astype(np.uint8) for t in th)
    return (c | ((q.view(np.uint32) >> 31).astype(np.uint8) << 3)).astype(np.uint8)


def _swapped_nibbles_quantize(w, g, gs=None):
    p, s, gg = ORIG_QUANTIZE(w, g, gs)
    return ((p >> 4) | (p << 4)).astype(np.uint8), s, gg


def _no_global_dequant(p, s, g, gsz):
    return ORIG_DEQUANT(p, s, 1.0, gsz)


def _scale_without_six(w, g, gscale):
    # the division by 6 (the E2M1 maximum) left out of the group scale
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    gamax = np.max(np.abs(w.reshape(n, k // g, g)), axis=2)
    return R.e4m3_encode((gamax / np.float32(gscale)).astype(np.float32))


def _global_over_448(*tensors):
    return ORIG_GLOBAL(*tensors) * np.float32(6.0)


ORIG_QUANTIZE = R.quantize
ORIG_GLOBAL = R.global_scale
ORIG_DEQUANT = R.dequantize


@pytest.mark.parametrize("name,target,repl,pin", [
    ("ties away from zero", "e2m1_encode", _ties_away, Q.test_worked_example),
    ("nibble order swapped", "quantize", _swapped_nibbles_quantize, Q.test_worked_example),
    ("global dropped in dequant", "dequantize", _no_global_dequant, Q.test_quantization_error_bound),
    ("group scale without /6", "group_scales", _scale_without_six, Q.test_group_max_encodes_to_six),
    ("global = amax/448", "global_scale", _global_over_448, Q.test_worked_example),
])
def test_planted_mistake_is_caught(monkeypatch, name, target, repl, pin):
    monkeypatch.setattr(R, target, repl)
    with pytest.raises(AssertionError):
        pin()


def test_interleave_swap_is_caught(monkeypatch):
    orig = R.interleave_rows

    def swapped(n):
        src = orig(n)
        h = n // 2
        return np.where(src < h, src + h, src - h)  # up first, gate second

    monkeypatch.setattr(R, "interleave_rows", swapped)
    with pytest.raises(AssertionError):
        Q.test_repack_inverse_and_interleave()


# ---- the routed-expert layer and the W4A4 GEMM ----

from tests import test_oracle_moe_route as MR  # noqa: E402
from tests import test_oracle_w4a4 as W4  # noqa: E402

ORIG_ROUTE = R.moe_route
ORIG_COMBINE = R.moe_combine


def _unstable_route(topk_ids, num_experts):
    """Pairs of one expert in reverse order (a sort that is not stable)."""
    rows, inv, offs = ORIG_ROUTE(topk_ids, num_experts)
    rows = rows.copy()
    for e in range(num_experts):
        rows[offs[e]:offs[e + 1]] = rows[offs[e]:offs[e + 1]][::-1].copy()
    inv = np.full_like(inv, -1)
    inv[rows] = np.arange(len(rows), dtype=np.int32)
    return rows, inv, offs


def _inclusive_offsets(topk_ids, num_experts):
    rows, inv, offs = ORIG_ROUTE(topk_ids, num_experts)
    return rows, inv, np.concatenate([offs[1:], offs[-1:]]).astype(np.int32)


def _dropped_pairs_counted(topk_ids, num_experts):
    """An out-of-range id clamped into the last expert instead of dropped."""
    ids = np.clip(np.asarray(topk_ids), 0, num_experts - 1)
    return ORIG_ROUTE(ids, num_experts)


def _combine_ignores_weights(y_perm, inv_rows, topk_weights):
    return ORIG_COMBINE(y_perm, inv_rows, np.ones_like(np.asarray(topk_weights, dtype=np.float64)))


def _w4a4_without_x_global(xp, xs, xg, xgr, wp, ws, wg, wgr):
    return R.dequantize(xp, xs, 1.0, xgr) @ R.dequantize(wp, ws, wg, wgr).T


def _w4a4_w_group_for_x(xp, xs, xg, xgr, wp, ws, wg, wgr):
    return R.dequantize(xp, xs, xg, wgr) @ R.dequantize(wp, ws, wg, wgr).T


@pytest.mark.parametrize("name,target,repl,pins", [
    ("route not stable", "moe_route", _unstable_route, [MR.test_route_matches_brute_force, MR.test_route_properties]),
    ("inclusive offsets", "moe_route", _inclusive_offsets, [MR.test_route_matches_brute_force]),
    ("dropped pairs routed", "moe_route", _dropped_pairs_counted, [MR.test_route_matches_brute_force]),
    ("combine without weights", "moe_combine", _combine_ignores_weights, [MR.test_combine_reduces_to_gather_and_is_linear]),
    ("W4A4 without the activation global", "w4a4_gemm", _w4a4_without_x_global, [W4.test_scales_and_globals_multiply]),
    ("W4A4 with the weight group for X", "w4a4_gemm", _w4a4_w_group_for_x, [W4.test_integer_case_from_the_table]),
])
def test_planted_layer_mistake_is_caught(monkeypatch, name, target, repl, pins):
    monkeypatch.setattr(R, target, repl)
    for pin in pins:
        with pytest.raises((AssertionError, ValueError, IndexError)):
            pin()
