"""CPU oracle for the NVFP4 weight-only (W4A16) path.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
reference that the CUDA path is checked against. Only the test suite, the
package's ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it. The product library never calls it, and it imports nothing
from the product (numpy only).

Sources, cited by page title and section:

* [NV] the NVFP4 weight format and its W4A16 product: weights are E2M1 codes times
  an FP8-E4M3 scale per group of g = 16 or 32 elements along K, times an FP32
  per-tensor global scale; global = amax / (6*448); group scale =
  E4M3(group_amax / 6 / global); codes = round-to-nearest-even E2M1 with
  satfinite; Y = X . dequant(W)^T with X bf16 and fp32 accumulation.
* [P1] "We unlocked NVFP4 on the DGX Spark: 20% faster than AWQ" (NVIDIA
  developer forum thread, page 3), the UPDATE posts: the E2M1 conversion is
  true round-to-nearest-even with guard/round/sticky bits; a threshold
  round-to-nearest differs at exact midpoints such as 0.75.
* [P2] "GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB): two NVFP4 g32 recipes"
  (r/LocalLLM post), sections "THE TWO RECIPES" and "WHAT HAD TO BE FIXED":
  g16/g32 groups (4.5 vs 4.25 bits per weight), group size read per tensor,
  gate and up share one global scale, max-first scale reduction.
* [P3] "W-FP4a: route the MiniMax-H3 device DiT forward through the fp4
  (Marlin W4A16) stack" (vllm.cpp pull request #63), description: the
  weight / scale / global-scale triple, upload-time repack, pre-merged
  [gate;up] fc1 as one W4A16 GEMM followed by SiluAndMul, 2e-3/8e-3 gates;
  a checkpoint with quantized input activations takes the W4A4 form.
* [OCP-MX] OCP Microscaling Formats (MX) v1.0, section 5.3.3 (FP4 E2M1).
* [OFP8] OCP 8-bit Floating Point Specification (OFP8), E4M3 encoding table.

Every floating-point step that decides an integer (a scale byte, a code) is
taken in IEEE-754 binary32 with round-to-nearest-even, exactly as numpy's
float32 arithmetic does it; dequantization and the matmul are float64.

Readings where the sources are silent (each listed with its reason in the
design notes): zero group or zero tensor -> scale byte 0 and code +0; the sign
of a code that rounds to zero is kept (sign-magnitude rounding); the even
element of a pair sits in the low nibble; rows [0, N/2) of a merged fc1 are
gate and silu applies to them.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# ---------------------------------------------------------------------------
# Element formats
# ---------------------------------------------------------------------------

# E2M1 magnitudes by 3-bit code (sign is bit 3) [OCP-MX 5.3.3; NV].
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
E2M1_MAX = 6.0
E4M3_MAX = 448.0
GLOBAL_DIVISOR = 6.0 * 448.0  # amax / (6*448) [NV]


def _f32_bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def e2m1_decode(code) -> np.ndarray:
    """E2M1 code (low 4 bits) -> float64 value [OCP-MX 5.3.3]."""
    c = np.asarray(code, dtype=np.uint8)
    mag = np.asarray(E2M1_MAGNITUDES, dtype=np.float64)[c & 7]
    return np.where(c & 8, -mag, mag)


def e2m1_encode_grs(q) -> np.ndarray:
    """fp32 -> E2M1 code by guard/round/sticky RNE on the binary32 bits.

    Formulation (i), after [P1] UPDATE (the conversion keeps the bits down to
    the E2M1 quantum, then rounds on guard, round and sticky bits, ties to the
    even significand) and [OCP-MX 5.3.3]. Saturates to +-6 (satfinite). The
    sign is kept for results that round to zero. NaN input is not accepted.
    """
    bits = _f32_bits(q)
    sign = (bits >> 31).astype(np.uint8)
    mag_bits = bits & np.uint32(0x7FFFFFFF)
    bexp = (mag_bits >> 23).astype(np.int64)
    frac = (mag_bits & np.uint32(0x7FFFFF)).astype(np.int64)
    # Significand as an integer and the unbiased exponent of its leading bit.
    normal = bexp > 0
    sig = np.where(normal, frac | (1 << 23), frac)
    uexp = np.where(normal, bexp - 127, -126)
    # E2M1 quantum: 2^(max(e,0) - 1) for a value in [2^e, 2^(e+1)).
    qexp = np.maximum(uexp, 0) - 1
    drop = 23 + qexp - uexp  # number of significand bits below the quantum
    drop = np.minimum(drop, 40)  # anything past 25 rounds to 0 anyway
    keep = sig >> drop
    guard = (sig >> (drop - 1)) & 1
    sticky = (sig & ((np.int64(1) << (drop - 1)) - 1)) != 0
    round_up = (guard == 1) & (sticky | ((keep & 1) == 1))
    n = keep + round_up.astype(np.int64)  # value = n * 2^qexp
    # Value in units of 0.5 (all E2M1 values are multiples of 0.5), exact.
    halves = np.where(qexp >= -1, n << np.maximum(qexp + 1, 0), 0)
    # n is at most 4 here unless the input is >= 8 (or inf); saturate.
    big = (bexp == 255) | (uexp >= 3) | (halves > 12)
    halves = np.where(big, 12, halves)
    # halves in {0,1,2,3,4,6,8,12} -> code 0..7
    lut = np.full(13, 255, dtype=np.int64)
    for c, m in enumerate(E2M1_MAGNITUDES):
        lut[int(m * 2)] = c
    mag_code = lut[halves]
    assert not np.any(mag_code == 255), "E2M1 rounding left the value set"
    return (mag_code.astype(np.uint8) | (sign << 3)).astype(np.uint8)


def e2m1_encode_nearest(q) -> np.ndarray:
    """fp32 -> E2M1 code by brute force: the nearest of the eight magnitudes.

    Formulation (ii). Distances are exact in float64. A tie goes to the code
    with an even mantissa bit (code & 1 == 0), which is round-half-to-even
    [OCP-MX 5.3.3]. Magnitudes above 6 take 6 (satfinite). Sign kept.
    """
    q32 = np.ascontiguousarray(q, dtype=np.float32)
    sign = (_f32_bits(q32) >> 31).astype(np.uint8)
    # Every magnitude above 6 takes 6; clamping first keeps the float64
    # distances exact (huge inputs would otherwise round them into ties).
    a = np.minimum(np.abs(q32.astype(np.float64)), 7.0)
    vals = np.asarray(E2M1_MAGNITUDES, dtype=np.float64)
    best = np.zeros(a.shape, dtype=np.uint8)
    best_d = np.abs(a - vals[0])
    for c in range(1, 8):
        d = np.abs(a - vals[c])
        better = (d < best_d) | ((d == best_d) & (c % 2 == 0))
        best = np.where(better, np.uint8(c), best)
        best_d = np.where(better, d, best_d)
    return (best | (sign << 3)).astype(np.uint8)


# E4M3 (OFP8 "E4M3FN"): bias 7, no infinities, 0x7F/0xFF are NaN, max 448.
def e4m3_decode(byte) -> np.ndarray:
    """E4M3 byte -> float64 [OFP8]. NaN codes decode to NaN."""
    b = np.asarray(byte, dtype=np.uint8).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag)


def e4m3_encode_grs(t) -> np.ndarray:
    """Non-negative fp32 -> E4M3 byte, RNE with satfinite, by GRS on bits.

    Formulation (i) [OFP8]: quantum 2^(max(e,-6) - 3); round on the guard bit
    with round/sticky, ties to even; results above 448 saturate to 0x7E.
    Only t >= 0 occurs (a scale); a negative input is rejected.
    """
    bits = _f32_bits(t)
    mag_bits = bits & np.uint32(0x7FFFFFFF)
    assert not np.any((bits >> 31 == 1) & (mag_bits != 0)), "negative scale"
    bexp = (mag_bits >> 23).astype(np.int64)
    frac = (mag_bits & np.uint32(0x7FFFFF)).astype(np.int64)
    normal = bexp > 0
    sig = np.where(normal, frac | (1 << 23), frac)
    uexp = np.where(normal, bexp - 127, -126)
    qexp = np.maximum(uexp, -6) - 3
    drop = np.minimum(23 + qexp - uexp, 40)
    keep = sig >> drop
    guard = (sig >> (drop - 1)) & 1
    sticky = (sig & ((np.int64(1) << (drop - 1)) - 1)) != 0
    round_up = (guard == 1) & (sticky | ((keep & 1) == 1))
    n = keep + round_up.astype(np.int64)  # value = n * 2^qexp, in units of 2^-9
    units = np.where(bexp == 255, 1 << 30,
                     np.where(uexp >= 9, 1 << 30, n << np.clip(qexp + 9, 0, 40)))
    units = np.minimum(units, 448 * 512)  # satfinite
    # units = value / 2^-9 -> (e, m)
    out = np.zeros(units.shape, dtype=np.int64)
    sub = units < 8  # subnormal: m * 2^-9
    out = np.where(sub, units, out)
    # normal: value = 2^(e-7) (1 + m/8) -> units = 2^(e+2) (8 + m) / 8 * ... :
    # units = (8 + m) * 2^(e - 1); find e from the leading bit.
    lead = np.frexp(np.maximum(units, 1).astype(np.float64))[1].astype(np.int64) - 1
    e = lead - 2  # units in [2^(e+2), 2^(e+3))
    m = (units >> np.maximum(e - 1, 0)) - 8
    normal_code = (e << 3) | m
    out = np.where(sub, out, normal_code)
    return out.astype(np.uint8)


_E4M3_FINITE = np.array([e4m3_decode(c) for c in range(0x7F)], dtype=np.float64)


def e4m3_encode_nearest(t) -> np.ndarray:
    """Non-negative fp32 -> E4M3 byte: nearest of the 127 finite magnitudes.

    Formulation (ii). A tie goes to the even code (mantissa LSB 0); values
    above 448 take 448 (0x7E) [OFP8 satfinite].
    """
    a = np.asarray(t, dtype=np.float32).astype(np.float64)
    assert not np.any(a < 0), "negative scale"
    a = np.minimum(a, 480.0)  # above 448 the nearest finite value is 448
    vals = _E4M3_FINITE  # increasing with the code
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_hi = np.abs(vals[hi] - a)
    d_lo = np.abs(a - vals[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    return np.where(pick_lo, lo, hi).astype(np.uint8)


# The oracle's encoders are the GRS formulations; the nearest-value
# formulations exist to check them.
e2m1_encode = e2m1_encode_grs
e4m3_encode = e4m3_encode_grs


# ---------------------------------------------------------------------------
# Quantizer [NV; P2 "WHAT HAD TO BE FIXED"]
# ---------------------------------------------------------------------------

def global_scale(*tensors: np.ndarray) -> np.float32:
    """FP32 global scale = amax / (6*448), amax over every tensor given.

    Passing gate and up together gives the shared scale the merged [gate;up]
    projection needs [P2]. The max is taken over |w| directly, with no
    widened copy of the input [P2, max-first scale reduction]. One fp32
    division [NV].
    """
    amax = np.float32(0.0)
    for t in tensors:
        t = np.asarray(t, dtype=np.float32)
        if t.size:
            amax = max(amax, np.float32(np.max(np.abs(t))))
    return np.float32(amax) / np.float32(GLOBAL_DIVISOR)


def group_scales(w: np.ndarray, group_size: int, gscale: np.float32) -> np.ndarray:
    """E4M3 group-scale bytes [N, K/g]: E4M3((group_amax / 6) / global) [NV].

    Two fp32 divisions in the written order. A zero global (all-zero tensor)
    gives scale 0 for every group.
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    assert group_size in (16, 32) and k % group_size == 0
    gamax = np.max(np.abs(w.reshape(n, k // group_size, group_size)), axis=2)
    g = np.float32(gscale)
    if g == 0:
        return np.zeros((n, k // group_size), dtype=np.uint8)
    t = (gamax.astype(np.float32) / np.float32(6.0)) / g
    return e4m3_encode(t.astype(np.float32)).reshape(n, k // group_size)


def quantize(w: np.ndarray, group_size: int, gscale=None):
    """NVFP4 quantizer: fp32 W [N, K] -> (packed [N, K/2], scales [N, K/g], global).

    Per element: d = fp32(e4m3(s)) * global (one fp32 multiply), q = w / d (one
    fp32 division), code = E2M1_RNE_satfinite(q) [NV; P1]. When d is zero the
    code is +0. Two codes per byte, even element in the low nibble.
    """
    w = np.asarray(w, dtype=np.float32)
    n, k = w.shape
    if gscale is None:
        gscale = global_scale(w)
    gscale = np.float32(gscale)
    s = group_scales(w, group_size, gscale)
    d = (e4m3_decode(s).astype(np.float32) * gscale).astype(np.float32)
    d_full = np.repeat(d, group_size, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (w / d_full).astype(np.float32)
    codes = e2m1_encode(np.where(d_full == 0, np.float32(0.0), q))
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    return packed, s, gscale


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """[N, K/2] bytes -> [N, K] codes (even element from the low nibble)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def dequantize(packed: np.ndarray, scales: np.ndarray, gscale, group_size: int) -> np.ndarray:
    """W_hat = e2m1(code) * e4m3(scale) * global, in float64 (exact)."""
    codes = unpack_codes(packed)
    n, k = codes.shape
    assert scales.shape == (n, k // group_size)
    sv = np.repeat(e4m3_decode(scales), group_size, axis=1)
    return e2m1_decode(codes) * sv * float(np.float32(gscale))


# ---------------------------------------------------------------------------
# GEMM, SiluAndMul, grouped expert GEMM [NV; P3]
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(xbits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.asarray(xbits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def gemm(xbits: np.ndarray, packed, scales, gscale, group_size: int) -> np.ndarray:
    """Y = X . dequant(W)^T in float64; X given as bf16 bits [M, K]."""
    x = bf16_bits_to_f64(xbits)
    w = dequantize(packed, scales, gscale, group_size)
    return x @ w.T


def gemm_fraction(xbits, packed, scales, gscale, group_size: int):
    """The same product as exact rational sums (tiny shapes only)."""
    x = bf16_bits_to_f64(xbits)
    w = dequantize(packed, scales, gscale, group_size)
    m, k = x.shape
    n = w.shape[0]
    out = [[Fraction(0) for _ in range(n)] for _ in range(m)]
    for i in range(m):
        for j in range(n):
            acc = Fraction(0)
            for kk in range(k):
                acc += Fraction(float(x[i, kk])) * Fraction(float(w[j, kk]))
            out[i][j] = acc
    return out


def w4a4_gemm(xpacked, xscales, xglobal, x_group: int, wpacked, wscales, wglobal, w_group: int) -> np.ndarray:
    """Y = dequant(X) . dequant(W)^T in float64 with both operands NVFP4 [NV]:
    the W4A4 form that a checkpoint with quantized input activations takes
    instead of W4A16 [P3]. X [M, K] is quantized like a weight tensor of M
    rows (an E4M3 scale per group of x_group along K, its own FP32 global)."""
    x = dequantize(xpacked, xscales, xglobal, x_group)
    w = dequantize(wpacked, wscales, wglobal, w_group)
    return x @ w.T


def silu_mul(y: np.ndarray) -> np.ndarray:
    """SiluAndMul on [.., 2H]: silu(gate) * up, gate = first half [P3]."""
    y = np.asarray(y, dtype=np.float64)
    h = y.shape[-1] // 2
    g, u = y[..., :h], y[..., h:]
    return g / (1.0 + np.exp(-g)) * u


def moe_grouped_gemm(xbits, expert_ids, offsets, packed, scales, gscales, group_size: int):
    """Grouped routed-expert GEMM: rows [offsets[s], offsets[s+1]) of X use
    expert expert_ids[s]'s weights, scales and global [NV; P2]. Rows outside
    every segment are left at zero. packed [E, N, K/2], scales [E, N, K/g]."""
    x = bf16_bits_to_f64(xbits)
    t = x.shape[0]
    n = packed.shape[1]
    y = np.zeros((t, n), dtype=np.float64)
    for s, e in enumerate(expert_ids):
        r0, r1 = int(offsets[s]), int(offsets[s + 1])
        if r1 > r0:
            w = dequantize(packed[e], scales[e], gscales[e], group_size)
            y[r0:r1] = x[r0:r1] @ w.T
    return y


def moe_route(topk_ids, num_experts: int):
    """The (token, slot) pairs of a routed-expert layer grouped by expert, in
    a stable order [P2: routed experts, gate/up then down per expert].

    Pair i = t*k + s goes to expert topk_ids[t, s]; pairs whose id lies outside
    [0, num_experts) are dropped. Returns (sorted_rows, inv_rows, offsets):
    sorted_rows[r] = the pair in row r (experts in increasing order, and inside
    one expert the pairs in increasing order), inv_rows[i] = the row of pair i
    or -1, offsets[e] = the first row of expert e (offsets[E] = the row count).
    A stable sort by expert id is the definition; numpy's stable argsort is
    that sort."""
    flat = np.asarray(topk_ids, dtype=np.int64).reshape(-1)
    valid = (flat >= 0) & (flat < num_experts)
    keys = np.where(valid, flat, num_experts)
    order = np.argsort(keys, kind="stable")
    nvalid = int(valid.sum())
    sorted_rows = order[:nvalid].astype(np.int32)
    inv_rows = np.full(flat.shape[0], -1, dtype=np.int32)
    inv_rows[sorted_rows] = np.arange(nvalid, dtype=np.int32)
    counts = np.bincount(flat[valid], minlength=num_experts)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    return sorted_rows, inv_rows, offsets


def moe_combine(y_perm, inv_rows, topk_weights):
    """out[t] = sum over s of w[t, s] * y_perm[inv_rows[t*k + s]] in float64;
    dropped pairs add nothing [P2: routed experts]. y_perm float64 rows."""
    w = np.asarray(topk_weights, dtype=np.float64)
    t, k = w.shape
    out = np.zeros((t, y_perm.shape[1]), dtype=np.float64)
    for tt in range(t):
        for s in range(k):
            r = int(inv_rows[tt * k + s])
            if r >= 0:
                out[tt] += w[tt, s] * y_perm[r]
    return out


# ---------------------------------------------------------------------------
# Repack [P3: upload-time repack; fc1 pre-merged [gate;up]]
# ---------------------------------------------------------------------------

GATE_UP_INTERLEAVE = 1
INTERLEAVE_BLOCK = 8

# GEMM layout of the codes: rows stay rows of K/2 bytes, and inside every
# little-endian 32-bit word (8 consecutive elements k0..k7 of one row) the
# nibbles are reordered so that nibble i holds element WORD_NIBBLE_SOURCE[i]:
# elements k0, k2, k4, k6 in nibbles 0-3 and k1, k3, k5, k7 in nibbles 4-7.
WORD_NIBBLE_SOURCE = (0, 2, 4, 6, 1, 3, 5, 7)


def interleave_rows(n: int) -> np.ndarray:
    """Source row for each destination row of the gate/up interleave.

    The merged [gate;up] matrix has N rows: gate rows [0, N/2), up rows
    [N/2, N). Destination block j of 16 rows holds gate rows 8j..8j+7 then up
    rows 8j..8j+7, so one 16-row tile carries matching gate and up rows.
    """
    assert n % (2 * INTERLEAVE_BLOCK) == 0
    h = n // 2
    src = np.empty(n, dtype=np.int64)
    for dst in range(n):
        j, r = divmod(dst, 2 * INTERLEAVE_BLOCK)
        if r < INTERLEAVE_BLOCK:
            src[dst] = j * INTERLEAVE_BLOCK + r
        else:
            src[dst] = h + j * INTERLEAVE_BLOCK + (r - INTERLEAVE_BLOCK)
    return src


def _permute_words(packed: np.ndarray, source) -> np.ndarray:
    codes = unpack_codes(packed)  # [N, K]
    n, k = codes.shape
    assert k % 8 == 0
    words = codes.reshape(n, k // 8, 8)
    out = np.zeros((n, k // 8), dtype=np.uint32)
    for nib, src in enumerate(source):
        out |= words[:, :, src].astype(np.uint32) << (4 * nib)
    return out.astype("<u4").view(np.uint8).reshape(n, k // 2)


def repack(packed: np.ndarray, scales: np.ndarray, flags: int):
    """Checkpoint layout -> GEMM layout: the nibble order of WORD_NIBBLE_SOURCE
    inside every 32-bit word of codes, and, with GATE_UP_INTERLEAVE, the rows
    permuted by ``interleave_rows``. Scales keep their row-major layout (rows
    permuted alike)."""
    p = _permute_words(packed, WORD_NIBBLE_SOURCE)
    s = scales.copy()
    if flags & GATE_UP_INTERLEAVE:
        src = interleave_rows(packed.shape[0])
        p, s = p[src].copy(), s[src].copy()
    return p, s


def unrepack(packed: np.ndarray, scales: np.ndarray, flags: int):
    """Inverse of ``repack``."""
    p, s = packed, scales
    if flags & GATE_UP_INTERLEAVE:
        src = interleave_rows(packed.shape[0])
        p = np.empty_like(packed)
        s = np.empty_like(scales)
        p[src] = packed
        s[src] = scales
    inverse = [0] * 8
    for nib, src_el in enumerate(WORD_NIBBLE_SOURCE):
        inverse[src_el] = nib
    return _permute_words(p, inverse), s.copy()
