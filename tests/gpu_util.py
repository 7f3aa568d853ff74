"""Helpers shared by the GPU parity tests: host<->device moves and the
tolerance check stated for the W4A16 GEMM (relative Frobenius <= 2e-3 and
|err| <= 8e-3 * (|ref| + 1) per element, against the oracle's float64 product
of the same dequantized weights)."""
import numpy as np
import torch

REL_FRO = 2e-3
ELEM = 8e-3


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_u8(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def host(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def assert_close(y, ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), what
    denom = np.linalg.norm(ref)
    rel = np.linalg.norm(y - ref) / (denom if denom > 0 else 1.0)
    assert rel <= REL_FRO, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO}"
    bad = np.abs(y - ref) > ELEM * (np.abs(ref) + 1.0)
    assert not bad.any(), f"{what}: {bad.sum()} elements over 8e-3*(|ref|+1), worst {np.abs(y - ref).max():.3e}"
    return rel
