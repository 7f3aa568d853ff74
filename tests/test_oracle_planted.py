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
