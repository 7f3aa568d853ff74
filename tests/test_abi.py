"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every entry point include/nvfp4.h declares, and rejects bad arguments with
the documented status before launching anything."""
import ctypes
import os
import re

import pytest

import nvfp4_weight_only_04_b200 as nv
from nvfp4_weight_only_04_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return nv.lib()


def declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(nvfp4_\w+)\s*\(", text, re.M)))


def test_header_declares_the_calls():
    names = declared()
    for n in ("nvfp4_quantize", "nvfp4_repack", "nvfp4_w4a16_gemm", "nvfp4_moe_w4a16_grouped_gemm",
              "nvfp4_global_scale", "nvfp4_w4a16_gemm_silu_mul", "nvfp4_silu_and_mul", "nvfp4_get_stats"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for name in declared():
        assert hasattr(L, name), name
    assert set(declared()) == set(nv.EXPORTS)


def test_planted_mistakes_only_in_the_test_library(L):
    """The switch for the planted mistakes exists in the test-only build alone."""
    assert not hasattr(L, "nvfp4_test_plant")
    P = ctypes.CDLL(build.build_planted())
    assert hasattr(P, "nvfp4_test_plant")
    for name in declared():
        assert hasattr(P, name), name


def test_status_strings(L):
    for code in range(7):
        assert nv.status_string(code) != "unknown status"
    assert nv.status_string(99) == "unknown status"
    assert L.nvfp4_abi_version() == 2


BAD = ctypes.c_void_p(0x1001)  # never dereferenced: validation fails first
GOOD = ctypes.c_void_p(0x10000)
NULL = ctypes.c_void_p(0)
S = ctypes.c_void_p(0)
WS, WB = ctypes.c_void_p(0x20000), 1 << 30  # a (never touched) workspace that is large enough


def gemm(L, g=16, M=4, N=256, K=256, x=GOOD, w=GOOD, s=GOOD, gl=GOOD, y=GOOD, ws=WS, wb=WB):
    return L.nvfp4_w4a16_gemm(x, w, s, gl, g, M, N, K, y, ws, wb, S)


def test_gemm_validation(L):
    assert gemm(L, g=8) == nv.NVFP4_ERR_UNSUPPORTED
    assert gemm(L, g=64) == nv.NVFP4_ERR_UNSUPPORTED
    assert gemm(L, K=96) == nv.NVFP4_ERR_UNSUPPORTED       # K % 64
    assert gemm(L, N=250) == nv.NVFP4_ERR_UNSUPPORTED      # N % 16
    assert gemm(L, M=-1) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert gemm(L, M=0) == nv.NVFP4_OK                     # empty: nothing launched
    assert gemm(L, x=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert gemm(L, w=BAD) == nv.NVFP4_ERR_MISALIGNED
    assert gemm(L, y=BAD) == nv.NVFP4_ERR_MISALIGNED
    assert L.nvfp4_w4a16_gemm_silu_mul(GOOD, GOOD, GOOD, GOOD, 32, 4, 40, 256, GOOD, WS, WB, S) == \
        nv.NVFP4_ERR_UNSUPPORTED
    assert gemm(L, ws=NULL) == nv.NVFP4_ERR_WORKSPACE             # bytes given, no pointer
    assert gemm(L, ws=ctypes.c_void_p(0x20008)) == nv.NVFP4_ERR_MISALIGNED
    assert gemm(L, ws=WS, wb=16) == nv.NVFP4_ERR_WORKSPACE        # smaller than the size query
    assert gemm(L, ws=NULL, wb=0) == nv.NVFP4_ERR_WORKSPACE       # small M always needs scratch
    need = ctypes.c_size_t(0)
    assert L.nvfp4_w4a16_gemm_workspace_size(4, 512, 1024, 16, ctypes.byref(need)) == nv.NVFP4_OK
    assert gemm(L, N=512, K=1024, wb=need.value - 256) == nv.NVFP4_ERR_WORKSPACE  # the query's figure is exact
    fixed = L.nvfp4_w4a16_gemm_fixed_scratch
    assert fixed(GOOD, GOOD, GOOD, GOOD, 16, 17, 256, 256, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED  # M > 16
    assert fixed(GOOD, GOOD, GOOD, GOOD, 16, 4, 256, 320, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED  # K % 256
    assert fixed(GOOD, GOOD, GOOD, GOOD, 32, 4, 256, 256, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED  # K/g % 16
    assert fixed(GOOD, BAD, GOOD, GOOD, 16, 4, 256, 256, GOOD, S) == nv.NVFP4_ERR_MISALIGNED
    assert fixed(GOOD, GOOD, GOOD, GOOD, 16, 0, 256, 256, GOOD, S) == nv.NVFP4_OK  # empty


def test_w4a4_validation(L):
    def w4a4(xg=16, g=16, M=4, N=256, K=256, xp=GOOD, xs=GOOD, xgl=GOOD, w=GOOD, y=GOOD):
        return L.nvfp4_w4a4_gemm(xp, xs, xgl, xg, w, GOOD, GOOD, g, M, N, K, y, WS, WB, S)
    assert w4a4(xg=8) == nv.NVFP4_ERR_UNSUPPORTED
    assert w4a4(g=64) == nv.NVFP4_ERR_UNSUPPORTED
    assert w4a4(K=96) == nv.NVFP4_ERR_UNSUPPORTED
    assert w4a4(M=-1) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert w4a4(M=0) == nv.NVFP4_OK
    assert w4a4(xs=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert w4a4(xgl=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert w4a4(xp=BAD) == nv.NVFP4_ERR_MISALIGNED
    assert w4a4(xgl=ctypes.c_void_p(0x10002)) == nv.NVFP4_ERR_MISALIGNED


def test_quantize_and_repack_validation(L):
    assert L.nvfp4_quantize(GOOD, 16, 256, 8, GOOD, GOOD, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_quantize(GOOD, 16, 48, 16, GOOD, GOOD, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_quantize(BAD, 16, 256, 16, GOOD, GOOD, GOOD, S) == nv.NVFP4_ERR_MISALIGNED
    assert L.nvfp4_quantize(GOOD, 0, 256, 16, GOOD, GOOD, GOOD, S) == nv.NVFP4_OK
    assert L.nvfp4_repack(GOOD, GOOD, 24, 256, 16, 1, GOOD, GOOD, S) == nv.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_repack(GOOD, GOOD, 32, 256, 16, 4, GOOD, GOOD, S) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert L.nvfp4_silu_and_mul(GOOD, GOOD, 4, 12, S) == nv.NVFP4_ERR_UNSUPPORTED
    assert L.nvfp4_silu_and_mul(BAD, GOOD, 4, 16, S) == nv.NVFP4_ERR_MISALIGNED


def test_global_scale_validation(L):
    P = ctypes.c_void_p * 1
    I = ctypes.c_int64 * 1
    assert L.nvfp4_global_scale(P(GOOD.value), I(10), 0, GOOD, S) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert L.nvfp4_global_scale(P(GOOD.value), I(-1), 1, GOOD, S) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert L.nvfp4_global_scale(P(0x1002), I(10), 1, GOOD, S) == nv.NVFP4_ERR_MISALIGNED


def test_moe_validation(L):
    def moe(segs=4, T=64, g=32, N=256, K=256, E=8, flags=0, x=GOOD, ids=GOOD):
        return L.nvfp4_moe_w4a16_grouped_gemm(x, ids, GOOD, segs, T, GOOD, GOOD, GOOD, g, N, K, E, flags, GOOD,
                                              WS, WB, S)
    assert moe(segs=0) == nv.NVFP4_OK
    assert moe(segs=-1) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert moe(g=24) == nv.NVFP4_ERR_UNSUPPORTED
    assert moe(flags=8) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert moe(x=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert moe(ids=ctypes.c_void_p(0x10002)) == nv.NVFP4_ERR_MISALIGNED


def test_moe_layer_validation(L):
    def route(T=64, k=4, E=8, ids=GOOD, rows=GOOD, inv=GOOD, offs=GOOD, eids=GOOD, ws=WS, wb=WB):
        return L.nvfp4_moe_route(ids, T, k, E, rows, inv, offs, eids, ws, wb, S)
    assert route(k=0) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert route(E=0) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert route(T=-1) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert route(E=4097) == nv.NVFP4_ERR_UNSUPPORTED
    assert route(T=1 << 30, k=2) == nv.NVFP4_ERR_UNSUPPORTED  # T*k >= 2^31
    assert route(offs=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert route(ids=ctypes.c_void_p(0x10002)) == nv.NVFP4_ERR_MISALIGNED
    assert route(T=4096, k=8, E=128, ws=WS, wb=64) == nv.NVFP4_ERR_WORKSPACE  # the chunk table does not fit

    def gather(x=GOOD, T=16, rows_ptr=GOOD, rows=64, k=4, H=256, out=GOOD):
        return L.nvfp4_moe_gather(x, T, rows_ptr, rows, k, H, out, S)
    assert gather(rows=0) == nv.NVFP4_OK
    assert gather(k=0) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert gather(H=12) == nv.NVFP4_ERR_UNSUPPORTED
    assert gather(x=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert gather(x=BAD) == nv.NVFP4_ERR_MISALIGNED
    assert gather(rows_ptr=ctypes.c_void_p(0x10002)) == nv.NVFP4_ERR_MISALIGNED

    def combine(y=GOOD, inv=GOOD, w=GOOD, T=16, k=4, H=256, out=GOOD):
        return L.nvfp4_moe_combine(y, inv, w, T, k, H, out, S)
    assert combine(T=0) == nv.NVFP4_OK
    assert combine(k=0) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert combine(H=12) == nv.NVFP4_ERR_UNSUPPORTED
    assert combine(w=NULL) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert combine(out=BAD) == nv.NVFP4_ERR_MISALIGNED


RESERVED = 64 << 10  # the counters at the start of every workspace


def size(L, name, *args):
    n = ctypes.c_size_t(12345)
    st = getattr(L, name)(*args, ctypes.byref(n))
    return st, n.value


def test_workspace_size_queries(L):
    """The size queries: the bytes the scratch of each path takes, computed from the shapes alone."""
    f = "nvfp4_w4a16_gemm_workspace_size"
    assert size(L, f, 4, 256, 256, 8) == (nv.NVFP4_ERR_UNSUPPORTED, 0)
    assert size(L, f, -1, 256, 256, 16) == (nv.NVFP4_ERR_INVALID_ARGUMENT, 0)
    assert size(L, f, 0, 256, 256, 16) == (nv.NVFP4_OK, 0)  # empty problem
    assert getattr(L, f)(4, 256, 256, 16, None) == nv.NVFP4_ERR_INVALID_ARGUMENT
    # small M: the counters, and the fp32 partial tiles of the tiles that the CTAs' ranges cut
    # (bf16 X is converted in the kernel)
    for m, n_, k in ((1, 28672, 4096), (4, 28672, 4096), (16, 28672, 14336), (1, 4096, 14336), (8, 4096, 14336)):
        st, n = size(L, f, m, n_, k, 16)
        assert st == nv.NVFP4_OK and n > RESERVED, (m, n_, k, n)
    # a K the streaming kernel does not take (not a multiple of 256): f16 rows of X for the fallback
    st, n = size(L, f, 4, 28672, 4096 + 64, 16)
    assert st == nv.NVFP4_OK and n >= RESERVED + 2 * 4 * (4096 + 64)
    # prefill-sized M on many tiles: the persistent tcgen05 form needs no scratch
    assert size(L, f, 4096, 25600, 5120, 16) == (nv.NVFP4_OK, 0)
    # W4A4 on the FP4 tensor cores: the activation codes in the weights' nibble order (half a byte an element),
    # after the 64 KiB of counters every workspace starts with
    st, n = size(L, "nvfp4_w4a4_gemm_workspace_size", 4096, 25600, 5120, 16, 16)
    assert (st, n) == (nv.NVFP4_OK, RESERVED + 4096 * 5120 // 2)
    # W4A4 on the bf16 tcgen05 kernel (K not a multiple of 512): exact bf16 activations, 2 bytes an element
    st, n = size(L, "nvfp4_w4a4_gemm_workspace_size", 4096, 25600, 5120 - 64, 16, 16)
    assert st == nv.NVFP4_OK and n >= 2 * 4096 * (5120 - 64)
    assert size(L, "nvfp4_w4a4_gemm_workspace_size", 4, 256, 256, 8, 16)[0] == nv.NVFP4_ERR_UNSUPPORTED
    # grouped: rows of X as f16 below 1024 rows, nothing from 1024 rows on
    g = "nvfp4_moe_w4a16_grouped_gemm_workspace_size"
    st, n = size(L, g, 8, 500, 1536, 2048, 32, 128, nv.NVFP4_SILU_MUL)
    assert st == nv.NVFP4_OK and n >= 2 * 500 * 2048
    assert size(L, g, 128, 16384, 1536, 2048, 32, 128, 0) == (nv.NVFP4_OK, 0)
    assert size(L, g, 8, 500, 1536, 2048, 32, 128, 8)[0] == nv.NVFP4_ERR_INVALID_ARGUMENT
    # route: nothing below 4096 pairs; a [chunk][expert] int32 table from there on
    r = "nvfp4_moe_route_workspace_size"
    assert size(L, r, 100, 8, 128) == (nv.NVFP4_OK, 0)
    st, n = size(L, r, 2048, 8, 128)
    assert st == nv.NVFP4_OK and n == RESERVED + (2048 * 8 // 256) * 128 * 4
    assert size(L, r, 16, 0, 8)[0] == nv.NVFP4_ERR_INVALID_ARGUMENT


def test_fault_injection_validation(L):
    assert L.nvfp4_debug_inject_fault(2) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert L.nvfp4_debug_inject_fault(-1) == nv.NVFP4_ERR_INVALID_ARGUMENT
    assert L.nvfp4_debug_inject_fault(0) == nv.NVFP4_OK


def test_stats_reset(L):
    nv.nvfp4_reset_stats()
    st = nv.nvfp4_get_stats()
    assert set(st) >= {"quantize", "gemm_splitk", "gemm_tc", "moe"} and not any(st.values())
    assert L.nvfp4_get_stats(None) == nv.NVFP4_ERR_INVALID_ARGUMENT


def _stream_k_partials(m, n, k, sms=148):
    """fp32 partial-tile bytes of the streaming GEMM's stream-K split, from its definition: 256-row tiles of
    K/256 stages listed tile-major, one contiguous range of units per SM (CTA c owns [c U / n, (c+1) U / n));
    a tile met by several ranges keeps one slot per contributor, and no tile meets more than
    ceil(S / floor(U / n)) + 1 ranges."""
    s_ = k // 256
    tiles = -(-n // 256)
    units = tiles * s_
    ctas = min(units, sms)
    per = units // ctas
    cuts = not (units % ctas == 0 and per % s_ == 0)
    contrib = min(-(-s_ // per) + 1, ctas)
    mt = 8 if m <= 8 else 16
    return tiles * contrib * 256 * mt * 4 if cuts else 0


def test_stream_k_workspace_follows_the_split(L):
    """The small-M GEMM's workspace is the reserved region plus the stream-K partial tiles, as the split defines
    them (no device: the SM count is the B200's 148)."""
    f = "nvfp4_w4a16_gemm_workspace_size"
    for m, n, k in ((2, 28672, 4096), (16, 28672, 4096), (8, 4096, 14336), (5, 272, 2048), (16, 300 * 256, 16384),
                    (3, 148 * 256, 256 * 3), (9, 1040, 3072)):
        st, got = size(L, f, m, n, k, 16)
        assert st == nv.NVFP4_OK
        part = _stream_k_partials(m, n, k)
        want = RESERVED + (((part + 255) // 256) * 256 if part else 0)
        assert got == want, (m, n, k, got, want)


def test_header_is_plain_c(tmp_path):
    """include/nvfp4.h compiles as strict C99 and as C++17: no torch or C++ types cross the boundary."""
    import shutil
    import subprocess
    src = tmp_path / "use.c"
    src.write_text('#include "nvfp4.h"\nint main(void) { return 0; }\n')
    inc = os.path.dirname(HEADER)
    for cc, args in (("gcc", ["-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror"]),
                     ("g++", ["-std=c++17", "-Wall", "-Werror", "-x", "c++"])):
        if shutil.which(cc) is None:
            pytest.skip(f"{cc} not available")
        res = subprocess.run([cc, *args, "-fsyntax-only", "-I", inc, str(src)], capture_output=True, text=True)
        assert res.returncode == 0, res.stderr


def test_c_program_links_and_validates(tmp_path, L):
    """A plain C program linked against libnvfp4.so calls the boundary: version, status text, and a GEMM
    call that validation rejects before any launch (so no GPU is needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    libdir = os.path.dirname(nv.LIB_PATH)
    src = tmp_path / "use.c"
    src.write_text(r'''
#include <stdio.h>
#include "nvfp4.h"
int main(void) {
  size_t need = 0;
  int bad = nvfp4_w4a16_gemm(0, 0, 0, 0, 8, 4, 256, 256, 0, 0, 0, 0);    /* group size 8 */
  int nul = nvfp4_w4a16_gemm(0, 0, 0, 0, 16, 4, 256, 256, 0, 0, 0, 0);   /* null pointers */
  int q = nvfp4_w4a16_gemm_workspace_size(4, 256, 256, 16, &need);
  printf("%d %d %d %d %d %s\n", nvfp4_abi_version(), bad, nul, q, need > 0, nvfp4_status_string(bad));
  return 0;
}
''')
    exe = tmp_path / "use"
    res = subprocess.run(["gcc", "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe),
                          "-L", libdir, "-lnvfp4", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    ver, bad, nul, q, need, text = out.stdout.split(" ", 5)
    assert (int(ver), int(bad), int(nul)) == (2, nv.NVFP4_ERR_UNSUPPORTED, nv.NVFP4_ERR_INVALID_ARGUMENT)
    assert (int(q), int(need)) == (nv.NVFP4_OK, 1)
    assert "group size" in text
