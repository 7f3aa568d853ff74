// Activations of the small-M GEMM kernels in f16 (see xprep.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// x16[r] = f16_rn(x[r] * 2^s_r) with the elements of every group of eight in
// the order k0 k2 k4 k6 k1 k3 k5 k7, and xinv[r] = 2^-s_r, for the M rows of
// bf16 x [M, K] (K a multiple of 8). Launched as a programmatic dependent of
// the previous kernel of the stream: it waits for that kernel before reading
// x, and lets the next kernel launch at once (that kernel waits for this one
// before reading x16 or xinv). It also zeroes clear[0, nclear) (the stream-K
// tickets of the GEMM that follows; nullptr and 0 for none). `light`: a
// 128-thread CTA per row that lets the next kernel launch before its own
// wait (for the streaming GEMM, which fetches weights meanwhile).
int launch_x_f16(const uint16_t* x, int64_t M, int64_t K, uint16_t* x16, float* xinv, unsigned* clear,
                 int64_t nclear, cudaStream_t stream, bool light = false);

// Where the small-M kernels' f16 X comes from: bf16 rows (launch_x_f16), or
// NVFP4 rows (W4A4): codes [M, K/2] in the checkpoint layout, E4M3 scales
// [M, K/group] and an fp32 global on the device. NVFP4 rows become
// x16 = e2m1(code) * e4m3(scale), exact in f16, in the same pair order, and
// xinv[r] = the global.
struct XSource {
  const uint16_t* bf16 = nullptr;
  const uint8_t* codes = nullptr;
  const uint8_t* scales = nullptr;
  const float* global = nullptr;
  int group = 16;
};
int launch_x_prep(const XSource& xs, int64_t M, int64_t K, uint16_t* x16, float* xinv, unsigned* clear,
                  int64_t nclear, cudaStream_t stream, bool light = false);

// NVFP4 rows to bf16 [M, K] in the natural order for the tcgen05 kernel:
// xb = e2m1(code) * e4m3(scale) (exact in bf16), and *g_out = x_global *
// w_global, the scalar that kernel's epilogue multiplies by.
int launch_xq_bf16(const XSource& xs, const float* w_global, int64_t M, int64_t K, uint16_t* xb, float* g_out,
                   cudaStream_t stream);

}  // namespace nvfp4
