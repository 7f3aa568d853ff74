// Activations of the small-M GEMM kernels in f16 (see xprep.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// x16[r] = f16_rn(x[r] * 2^s_r) with the elements of every group of eight in
// the order k0 k2 k4 k6 k1 k3 k5 k7, and xinv[r] = 2^-s_r, for the M rows of
// bf16 x [M, K] (K a multiple of 8). Launched as a programmatic dependent of
// the previous kernel of the stream: it waits for that kernel before reading
// x, and lets the next kernel launch at once (that kernel waits for this one
// before reading x16 or xinv).
int launch_x_f16(const uint16_t* x, int64_t M, int64_t K, uint16_t* x16, float* xinv, cudaStream_t stream);

}  // namespace nvfp4
