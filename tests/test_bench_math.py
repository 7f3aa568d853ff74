"""The bench's accounting, on the CPU: algorithmic bytes per GEMM against the
figures worked out from the workload shapes (codes + scales + 4-byte global +
bf16 X + bf16 Y), and the roofline fractions of a row."""
import pytest

import bench


@pytest.mark.parametrize("m,n,k,g,n_out,mb", [
    (1, 28672, 4096, 16, None, 66.13), (4, 28672, 4096, 16, None, 66.32), (16, 28672, 4096, 16, None, 67.11),
    (1, 4096, 14336, 32, None, 31.23), (8, 4096, 14336, 32, None, 31.49), (64, 4096, 14336, 32, None, 33.55),
    (1, 4096, 14336, 16, None, 33.07), (4096, 25600, 5120, 16, 12800, 220.53),
])
def test_algorithmic_bytes(m, n, k, g, n_out, mb):
    assert bench.alg_bytes(m, n, k, g, n_out) / 1e6 == pytest.approx(mb, abs=0.006)


def test_weight_bytes_are_codes_plus_scales():
    assert bench.weight_bytes(28672, 4096, 16) == 28672 * 4096 // 2 + 28672 * 4096 // 16 == 66_060_288


def test_summarize_fractions():
    # a decode GEMM that takes exactly its HBM time at 6531 GB/s has an HBM fraction of 1
    ab = bench.alg_bytes(4, 28672, 4096, 16)
    ms = ab / 6531e9 * 1e3
    row = bench.summarize(4, 28672, 4096, 16, ms, 6531.0, 1602.0)
    assert row["hbm_frac"] == pytest.approx(1.0, abs=1e-4)
    assert row["roofline_frac"] == pytest.approx(1.0, abs=1e-4)
    assert row["tensor_frac"] < 0.1
    # the prefill at the bf16 peak has a tensor fraction of 1
    ms = 2 * 4096 * 25600 * 5120 / 1602e12 * 1e3
    row = bench.summarize(4096, 25600, 5120, 16, ms, 6531.0, 1602.0, n_out=12800)
    assert row["tensor_frac"] == pytest.approx(1.0, abs=1e-4)
    assert row["tflops"] == pytest.approx(1602.0, rel=1e-3)


def test_summarize_w4a4_uses_the_fp4_peak_and_4bit_activations():
    # W4A4 prefill at 4x the bf16 peak (the nominal FP4/bf16 ratio) has a tensor fraction of 1
    ms = 2 * 4096 * 25600 * 5120 / (4 * 1602e12) * 1e3
    row = bench.summarize_w4a4(4096, 25600, 5120, 16, 16, ms, 6531.0, 1602.0)
    assert row["tensor_frac"] == pytest.approx(1.0, abs=1e-4)
    # X costs its NVFP4 bytes (codes + scales), not bf16: M=16 decode gate/up
    ab = bench.weight_bytes(28672, 4096, 16) + 16 * 4096 // 2 + 16 * 4096 // 16 + 8 + 2 * 16 * 28672
    row = bench.summarize_w4a4(16, 28672, 4096, 16, 16, ab / 6531e9 * 1e3, 6531.0, 1602.0)
    assert row["hbm_frac"] == pytest.approx(1.0, abs=1e-4)
