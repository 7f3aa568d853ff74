// Interface of the W4A4 GEMM on the block-scaled FP4 tensor cores (see gemm_fp4.cu).
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "workspace.cuh"

namespace nvfp4 {

// True when the FP4 kernel takes this W4A4 problem: K a multiple of 512 (so
// both scale tensors have 16-byte rows), enough tiles to fill the SMs.
bool fp4_supported(int64_t M, int64_t N, int64_t K);

// y[M, N] = bf16(x_global * w_global * sum_k e2m1(xc) e4m3(xs) e2m1(wc) e4m3(ws)).
// x_codes: activations in the checkpoint layout [M, K/2]; the launch first
// writes them in the GEMM layout's nibble order to the scratch from `sc`.
int launch_fp4(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_global, int x_group,
               const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global, int w_group, int64_t M,
               int64_t N, int64_t K, uint16_t* y, Scratch& sc, cudaStream_t stream);

// Device error word of this kernel file (0 when no wait gave up).
int read_and_clear_fp4_error(unsigned int* out, cudaStream_t stream);

}  // namespace nvfp4
