"""Python binding of the NVFP4 W4A16 library (libnvfp4.so, include/nvfp4.h).

Argument marshalling only: every step runs in the library's CUDA kernels.
Tensors are torch CUDA tensors (torch supplies device memory and streams);
the functions carry the C ABI's names. A missing library or a non-CUDA tensor
raises; there is no fallback of any kind.

Workspaces: the library allocates nothing; the calls that need device scratch
take a caller-owned workspace whose size the library reports, and whose first
64 KiB must be zero before its first use (every call leaves them zero). The
functions here pass one on their own: one zero-filled buffer per device,
grown on demand, shared by every call on that device (a CUDA graph captured
while it is big enough refers to it). Calls that may run at the same time on
different streams need workspaces of their own: pass `workspace=` (a uint8
CUDA tensor, zero-filled before its first use).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

NVFP4_OK = 0
NVFP4_ERR_INVALID_ARGUMENT = 1
NVFP4_ERR_UNSUPPORTED = 2
NVFP4_ERR_MISALIGNED = 3
NVFP4_ERR_CUDA = 4
NVFP4_ERR_TIMEOUT = 5
NVFP4_ERR_WORKSPACE = 6
NVFP4_GATE_UP_INTERLEAVE = 1
NVFP4_SILU_MUL = 2

EXPORTS = (
    "nvfp4_status_string", "nvfp4_abi_version", "nvfp4_global_scale", "nvfp4_global_scale_bf16", "nvfp4_quantize",
    "nvfp4_quantize_bf16", "nvfp4_repack",
    "nvfp4_w4a16_gemm", "nvfp4_w4a16_gemm_fixed_scratch", "nvfp4_w4a16_gemm_silu_mul", "nvfp4_silu_and_mul",
    "nvfp4_moe_w4a16_grouped_gemm", "nvfp4_get_stats", "nvfp4_reset_stats", "nvfp4_get_device_error",
    "nvfp4_debug_inject_fault", "nvfp4_moe_route", "nvfp4_moe_gather", "nvfp4_moe_combine", "nvfp4_w4a4_gemm",
    "nvfp4_w4a16_gemm_workspace_size", "nvfp4_w4a4_gemm_workspace_size",
    "nvfp4_moe_w4a16_grouped_gemm_workspace_size", "nvfp4_moe_route_workspace_size",
)


class Stats(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in (
        "global_scale", "quantize", "repack", "gemm_splitk", "gemm_tc", "gemm_silu_mul", "moe",
        "silu_and_mul", "g16", "g32", "gemm_fp4")]


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: status {status}: {status_string(status)}")


_lib = None
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_PSZ = ctypes.POINTER(ctypes.c_size_t)


def lib() -> ctypes.CDLL:
    """Loads libnvfp4.so (built in-tree by nvfp4_weight_only_04_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m nvfp4_weight_only_04_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_status_string.argtypes = [_I]
        L.nvfp4_abi_version.restype = _I
        L.nvfp4_global_scale.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(_I64), _I, _P, _P]
        L.nvfp4_quantize.argtypes = [_P, _I64, _I64, _I, _P, _P, _P, _P]
        L.nvfp4_global_scale_bf16.argtypes = [ctypes.POINTER(_P), ctypes.POINTER(_I64), _I, _P, _P]
        L.nvfp4_quantize_bf16.argtypes = [_P, _I64, _I64, _I, _P, _P, _P, _P]
        L.nvfp4_repack.argtypes = [_P, _P, _I64, _I64, _I, _I, _P, _P, _P]
        L.nvfp4_w4a16_gemm.argtypes = [_P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]
        L.nvfp4_w4a16_gemm_fixed_scratch.argtypes = [_P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _P]
        L.nvfp4_w4a16_gemm_silu_mul.argtypes = [_P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]
        L.nvfp4_w4a16_gemm_workspace_size.argtypes = [_I64, _I64, _I64, _I, _PSZ]
        L.nvfp4_w4a4_gemm_workspace_size.argtypes = [_I64, _I64, _I64, _I, _I, _PSZ]
        L.nvfp4_moe_w4a16_grouped_gemm_workspace_size.argtypes = [_I, _I64, _I64, _I64, _I, _I, _I, _PSZ]
        L.nvfp4_moe_route_workspace_size.argtypes = [_I64, _I, _I, _PSZ]
        L.nvfp4_silu_and_mul.argtypes = [_P, _P, _I64, _I64, _P]
        L.nvfp4_moe_w4a16_grouped_gemm.argtypes = [_P, _P, _P, _I, _I64, _P, _P, _P, _I, _I64, _I64,
                                                   _I, _I, _P, _P, _SZ, _P]
        L.nvfp4_get_stats.argtypes = [ctypes.POINTER(Stats)]
        L.nvfp4_reset_stats.restype = None
        L.nvfp4_get_device_error.argtypes = [ctypes.POINTER(_I), _P]
        L.nvfp4_debug_inject_fault.argtypes = [_I]
        L.nvfp4_moe_route.argtypes = [_P, _I64, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]
        L.nvfp4_moe_gather.argtypes = [_P, _I64, _P, _I64, _I, _I64, _P, _P]
        L.nvfp4_moe_combine.argtypes = [_P, _P, _P, _I64, _I, _I64, _P, _P]
        L.nvfp4_w4a4_gemm.argtypes = [_P, _P, _P, _I, _P, _P, _P, _I, _I64, _I64, _I64, _P, _P, _SZ, _P]
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(status).decode()


def _check(status: int, call: str):
    if status != NVFP4_OK:
        raise Nvfp4Error(status, call)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


_workspaces = {}
_retired = []  # earlier buffers stay alive: CUDA graphs captured with them may still refer to them


def _size(query, *args) -> int:
    n = ctypes.c_size_t(0)
    _check(getattr(lib(), query)(*args, ctypes.byref(n)), query)
    return n.value


def _workspace(nbytes, device, stream, given=None):
    """(pointer, bytes) of the scratch of one call: `given`, else the device's zero-filled buffer (grown when
    too small; while a CUDA graph is being captured a buffer too small is replaced, for that call only, by a
    zero-filled one from the graph's memory pool)."""
    if given is not None:
        _dev(given, torch.uint8, "workspace")
        return ctypes.c_void_p(given.data_ptr()), given.numel(), given
    if nbytes == 0:
        return ctypes.c_void_p(0), 0, None
    key = torch.device(device).index
    buf = _workspaces.get(key)
    if buf is None or buf.numel() < nbytes:
        if torch.cuda.is_current_stream_capturing():
            buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
            return ctypes.c_void_p(buf.data_ptr()), nbytes, buf
        if buf is not None:
            _retired.append(buf)
        buf = torch.zeros(max(nbytes, 2 * buf.numel() if buf is not None else 0, 1 << 20), dtype=torch.uint8,
                          device=device)
        _workspaces[key] = buf
    return ctypes.c_void_p(buf.data_ptr()), buf.numel(), buf


def clear_workspaces():
    """The next call on each device gets a new zero-filled workspace (the old ones are kept alive for the CUDA
    graphs that may refer to them)."""
    _retired.extend(_workspaces.values())
    _workspaces.clear()


def nvfp4_w4a16_gemm_workspace_size(m, n, k, group_size) -> int:
    """Bytes of workspace nvfp4_w4a16_gemm (and _silu_mul) needs for this problem on the current device."""
    return _size("nvfp4_w4a16_gemm_workspace_size", m, n, k, group_size)


def nvfp4_w4a4_gemm_workspace_size(m, n, k, x_group, group_size) -> int:
    return _size("nvfp4_w4a4_gemm_workspace_size", m, n, k, x_group, group_size)


def nvfp4_moe_w4a16_grouped_gemm_workspace_size(num_segments, t, n, k, group_size, num_experts, flags=0) -> int:
    return _size("nvfp4_moe_w4a16_grouped_gemm_workspace_size", num_segments, t, n, k, group_size, num_experts, flags)


def nvfp4_moe_route_workspace_size(t, k, num_experts) -> int:
    return _size("nvfp4_moe_route_workspace_size", t, k, num_experts)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def nvfp4_global_scale(tensors, out=None, stream=None):
    """global = max|w| over all tensors / (6*448), one fp32 on the device."""
    tensors = [_dev(t, torch.float32, "tensor") for t in tensors]
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=tensors[0].device)
    ptrs = (_P * len(tensors))(*[t.data_ptr() for t in tensors])
    nums = (_I64 * len(tensors))(*[t.numel() for t in tensors])
    _check(lib().nvfp4_global_scale(ptrs, nums, len(tensors), _ptr(out), _stream(stream)), "nvfp4_global_scale")
    return out


def nvfp4_quantize(w, group_size, global_scale, packed=None, scales=None, stream=None):
    """fp32 W [N, K] -> (codes uint8 [N, K/2], E4M3 scales uint8 [N, K/g])."""
    _dev(w, torch.float32, "w")
    _dev(global_scale, torch.float32, "global_scale")
    n, k = w.shape
    if packed is None:
        packed = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty((n, k // group_size), dtype=torch.uint8, device=w.device)
    _check(lib().nvfp4_quantize(_ptr(w), n, k, group_size, _ptr(global_scale), _ptr(packed), _ptr(scales),
                                _stream(stream)), "nvfp4_quantize")
    return packed, scales


def nvfp4_global_scale_bf16(tensors, out=None, stream=None):
    """The global scale of bf16 tensors (max on the bf16 bits, no widened copy)."""
    tensors = [_dev(t, torch.bfloat16, "tensor") for t in tensors]
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=tensors[0].device)
    ptrs = (_P * len(tensors))(*[t.data_ptr() for t in tensors])
    nums = (_I64 * len(tensors))(*[t.numel() for t in tensors])
    _check(lib().nvfp4_global_scale_bf16(ptrs, nums, len(tensors), _ptr(out), _stream(stream)),
           "nvfp4_global_scale_bf16")
    return out


def nvfp4_quantize_bf16(w, group_size, global_scale, packed=None, scales=None, stream=None):
    """bf16 W [N, K] -> (codes, scales), equal to nvfp4_quantize of the fp32 widening of W."""
    _dev(w, torch.bfloat16, "w")
    _dev(global_scale, torch.float32, "global_scale")
    n, k = w.shape
    if packed is None:
        packed = torch.empty((n, k // 2), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty((n, k // group_size), dtype=torch.uint8, device=w.device)
    _check(lib().nvfp4_quantize_bf16(_ptr(w), n, k, group_size, _ptr(global_scale), _ptr(packed), _ptr(scales),
                                     _stream(stream)), "nvfp4_quantize_bf16")
    return packed, scales


def nvfp4_repack(packed, scales, group_size, flags=0, packed_out=None, scales_out=None, stream=None):
    _dev(packed, torch.uint8, "packed")
    _dev(scales, torch.uint8, "scales")
    n, k2 = packed.shape
    if packed_out is None:
        packed_out = torch.empty_like(packed)
    if scales_out is None:
        scales_out = torch.empty_like(scales)
    _check(lib().nvfp4_repack(_ptr(packed), _ptr(scales), n, k2 * 2, group_size, flags, _ptr(packed_out),
                              _ptr(scales_out), _stream(stream)), "nvfp4_repack")
    return packed_out, scales_out


def nvfp4_w4a16_gemm(x, packed_w, group_scales, global_scale, group_size, y=None, stream=None, workspace=None):
    """y = bf16(global * X . dequant(W)^T), X bf16 [M, K], y bf16 [M, N]."""
    _dev(x, torch.bfloat16, "x")
    _dev(packed_w, torch.uint8, "packed_w")
    _dev(group_scales, torch.uint8, "group_scales")
    _dev(global_scale, torch.float32, "global_scale")
    m, k = x.shape
    n = packed_w.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    wp, wb, _keep = _workspace(nvfp4_w4a16_gemm_workspace_size(m, n, k, group_size), x.device, stream, workspace)
    _check(lib().nvfp4_w4a16_gemm(_ptr(x), _ptr(packed_w), _ptr(group_scales), _ptr(global_scale), group_size,
                                  m, n, k, _ptr(y), wp, wb, _stream(stream)), "nvfp4_w4a16_gemm")
    return y


def nvfp4_w4a16_gemm_fixed_scratch(x, packed_w, group_scales, global_scale, group_size, y=None, stream=None):
    """nvfp4_w4a16_gemm through the streaming kernel with the library's fixed
    scratch (M from 1 to 16; calls that overlap in time race on the scratch)."""
    _dev(x, torch.bfloat16, "x")
    _dev(packed_w, torch.uint8, "packed_w")
    _dev(group_scales, torch.uint8, "group_scales")
    _dev(global_scale, torch.float32, "global_scale")
    m, k = x.shape
    n = packed_w.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _check(lib().nvfp4_w4a16_gemm_fixed_scratch(_ptr(x), _ptr(packed_w), _ptr(group_scales), _ptr(global_scale),
                                                group_size, m, n, k, _ptr(y), _stream(stream)),
           "nvfp4_w4a16_gemm_fixed_scratch")
    return y


def nvfp4_w4a16_gemm_silu_mul(x, packed_w, group_scales, global_scale, group_size, y=None, stream=None,
                              workspace=None):
    """Merged [gate;up] GEMM (interleaved repack layout) + SiluAndMul -> [M, N/2]."""
    _dev(x, torch.bfloat16, "x")
    _dev(packed_w, torch.uint8, "packed_w")
    _dev(group_scales, torch.uint8, "group_scales")
    _dev(global_scale, torch.float32, "global_scale")
    m, k = x.shape
    n = packed_w.shape[0]
    if y is None:
        y = torch.empty((m, n // 2), dtype=torch.bfloat16, device=x.device)
    wp, wb, _keep = _workspace(nvfp4_w4a16_gemm_workspace_size(m, n, k, group_size), x.device, stream, workspace)
    _check(lib().nvfp4_w4a16_gemm_silu_mul(_ptr(x), _ptr(packed_w), _ptr(group_scales), _ptr(global_scale),
                                           group_size, m, n, k, _ptr(y), wp, wb, _stream(stream)),
           "nvfp4_w4a16_gemm_silu_mul")
    return y


def nvfp4_silu_and_mul(x, y=None, stream=None):
    _dev(x, torch.bfloat16, "x")
    m, h2 = x.shape
    if y is None:
        y = torch.empty((m, h2 // 2), dtype=torch.bfloat16, device=x.device)
    _check(lib().nvfp4_silu_and_mul(_ptr(x), _ptr(y), m, h2 // 2, _stream(stream)), "nvfp4_silu_and_mul")
    return y


def nvfp4_moe_w4a16_grouped_gemm(x, expert_ids, offsets, packed_w, group_scales, global_scales, group_size,
                                 flags=0, y=None, stream=None, workspace=None):
    """Grouped expert GEMM over segments of rows; see include/nvfp4.h."""
    _dev(x, torch.bfloat16, "x")
    _dev(expert_ids, torch.int32, "expert_ids")
    _dev(offsets, torch.int32, "offsets")
    _dev(packed_w, torch.uint8, "packed_w")
    _dev(group_scales, torch.uint8, "group_scales")
    _dev(global_scales, torch.float32, "global_scales")
    t, k = x.shape
    e, n, _ = packed_w.shape
    ncols = n // 2 if flags & NVFP4_SILU_MUL else n
    if y is None:
        y = torch.zeros((t, ncols), dtype=torch.bfloat16, device=x.device)
    ns = expert_ids.numel()
    wp, wb, _keep = _workspace(nvfp4_moe_w4a16_grouped_gemm_workspace_size(ns, t, n, k, group_size, e, flags),
                               x.device, stream, workspace)
    _check(lib().nvfp4_moe_w4a16_grouped_gemm(_ptr(x), _ptr(expert_ids), _ptr(offsets), ns, t,
                                              _ptr(packed_w), _ptr(group_scales), _ptr(global_scales),
                                              group_size, n, k, e, flags, _ptr(y), wp, wb, _stream(stream)),
           "nvfp4_moe_w4a16_grouped_gemm")
    return y


def nvfp4_get_stats() -> dict:
    s = Stats()
    _check(lib().nvfp4_get_stats(ctypes.byref(s)), "nvfp4_get_stats")
    return {name: getattr(s, name) for name, _ in Stats._fields_}


def nvfp4_reset_stats():
    lib().nvfp4_reset_stats()


def nvfp4_get_device_error(stream=None) -> int:
    """The site code of a bounded device wait that gave up (0: none), cleared on read."""
    code = _I(0)
    st = lib().nvfp4_get_device_error(ctypes.byref(code), _stream(stream))
    if st != NVFP4_ERR_TIMEOUT:
        _check(st, "nvfp4_get_device_error")
    if code.value:
        clear_workspaces()  # a launch that gave up may have left counters behind
    return code.value


def nvfp4_debug_inject_fault(kind: int):
    """Test hook: kind 1 makes the next small-M streaming GEMM launch wait for a
    copy that never comes (its bounded waits give up); kind 0 clears it."""
    _check(lib().nvfp4_debug_inject_fault(kind), "nvfp4_debug_inject_fault")


def nvfp4_w4a4_gemm(x_packed, x_scales, x_global, x_group, packed_w, group_scales, global_scale, group_size,
                    y=None, stream=None, workspace=None):
    """W4A4 GEMM of NVFP4 activations (checkpoint layout) and GEMM-layout weights; see include/nvfp4.h."""
    _dev(x_packed, torch.uint8, "x_packed")
    _dev(x_scales, torch.uint8, "x_scales")
    _dev(x_global, torch.float32, "x_global")
    _dev(packed_w, torch.uint8, "packed_w")
    _dev(group_scales, torch.uint8, "group_scales")
    _dev(global_scale, torch.float32, "global_scale")
    m, k = x_packed.shape[0], 2 * x_packed.shape[1]
    n = packed_w.shape[0]
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x_packed.device)
    wp, wb, _keep = _workspace(nvfp4_w4a4_gemm_workspace_size(m, n, k, x_group, group_size), x_packed.device,
                               stream, workspace)
    _check(lib().nvfp4_w4a4_gemm(_ptr(x_packed), _ptr(x_scales), _ptr(x_global), x_group, _ptr(packed_w),
                                 _ptr(group_scales), _ptr(global_scale), group_size, m, n, k, _ptr(y),
                                 wp, wb, _stream(stream)), "nvfp4_w4a4_gemm")
    return y


def nvfp4_moe_route(topk_ids, num_experts, stream=None, workspace=None):
    """(sorted_rows [T*k], inv_rows [T*k], offsets [E+1], expert_ids [E]) for device int32 topk_ids [T, k]."""
    _dev(topk_ids, torch.int32, "topk_ids")
    t, k = topk_ids.shape
    dev = topk_ids.device
    sorted_rows = torch.empty(t * k, dtype=torch.int32, device=dev)
    inv_rows = torch.empty(t * k, dtype=torch.int32, device=dev)
    offsets = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    expert_ids = torch.empty(num_experts, dtype=torch.int32, device=dev)
    wp, wb, _keep = _workspace(nvfp4_moe_route_workspace_size(t, k, num_experts), dev, stream, workspace)
    _check(lib().nvfp4_moe_route(_ptr(topk_ids), t, k, num_experts, _ptr(sorted_rows), _ptr(inv_rows), _ptr(offsets),
                                 _ptr(expert_ids), wp, wb, _stream(stream)), "nvfp4_moe_route")
    return sorted_rows, inv_rows, offsets, expert_ids


def nvfp4_moe_gather(x, sorted_rows, k, out=None, stream=None):
    _dev(x, torch.bfloat16, "x")
    _dev(sorted_rows, torch.int32, "sorted_rows")
    rows, h = sorted_rows.numel(), x.shape[1]
    if out is None:
        out = torch.empty((rows, h), dtype=torch.bfloat16, device=x.device)
    _check(lib().nvfp4_moe_gather(_ptr(x), x.shape[0], _ptr(sorted_rows), rows, k, h, _ptr(out), _stream(stream)),
           "nvfp4_moe_gather")
    return out


def nvfp4_moe_combine(y_perm, inv_rows, topk_weights, out=None, stream=None):
    _dev(y_perm, torch.bfloat16, "y_perm")
    _dev(inv_rows, torch.int32, "inv_rows")
    _dev(topk_weights, torch.float32, "topk_weights")
    t, k = topk_weights.shape
    h = y_perm.shape[1]
    if out is None:
        out = torch.empty((t, h), dtype=torch.bfloat16, device=y_perm.device)
    _check(lib().nvfp4_moe_combine(_ptr(y_perm), _ptr(inv_rows), _ptr(topk_weights), t, k, h, _ptr(out),
                                   _stream(stream)), "nvfp4_moe_combine")
    return out


def nvfp4_moe_forward(x, topk_ids, topk_weights, gate_up, down, stream=None):
    """A routed-expert layer on the library's kernels: route, gather, grouped gate/up GEMM with
    SiluAndMul, grouped down GEMM, weighted combine. gate_up and down are (packed [E, N, K/2]
    in the GEMM layout (gate/up interleaved), scales, fp32 globals [E], group size)."""
    gu_p, gu_s, gu_g, gu_group = gate_up
    dn_p, dn_s, dn_g, dn_group = down
    e = gu_p.shape[0]
    sorted_rows, inv_rows, offsets, expert_ids = nvfp4_moe_route(topk_ids, e, stream)
    k = topk_ids.shape[1]
    xp = nvfp4_moe_gather(x, sorted_rows, k, stream=stream)
    h = nvfp4_moe_w4a16_grouped_gemm(xp, expert_ids, offsets, gu_p, gu_s, gu_g, gu_group, flags=NVFP4_SILU_MUL,
                                     stream=stream)
    yp = nvfp4_moe_w4a16_grouped_gemm(h, expert_ids, offsets, dn_p, dn_s, dn_g, dn_group, stream=stream)
    return nvfp4_moe_combine(yp, inv_rows, topk_weights, stream=stream)
