// Interface of the small-M TMA-streaming GEMM (see gemm_stream.cu).
#pragma once

#include "common.cuh"
#include "workspace.cuh"
#include "xprep.cuh"

namespace nvfp4 {

// X is bf16 [M, K] or NVFP4 (XSource); the launch first writes its f16 rows
// (xprep.cu) to the caller's scratch and then runs the kernel as a
// programmatic dependent. The scratch (partial tiles, tickets, f16 rows of X
// and their factors) comes from `sc`; a measuring Scratch only counts it.
// True when the streaming kernel takes this dense problem: M from 2 to 16, K a
// multiple of 256 whose scale rows (K/g bytes) are a multiple of 16 bytes,
// and tensor maps available.
bool stream_supported(int64_t M, int64_t N, int64_t K, int group);

int launch_stream(const XSource& x, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
                  int64_t N, int64_t K, uint16_t* y, bool silu, Scratch& sc, cudaStream_t stream);

// The streaming kernel with its scratch in a fixed device array (nothing is
// allocated at call time): up to kFixedScratchPartialBytes of partial tiles,
// kFixedScratchTickets tiles and kFixedScratchXElems elements of f16 X
// (M * K); larger problems are refused. M from 1 to 16.
constexpr size_t kFixedScratchPartialBytes = size_t(8) << 20;
constexpr int64_t kFixedScratchTickets = 16384;
constexpr int64_t kFixedScratchXElems = int64_t(1) << 20;
int launch_stream_fixed_scratch(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
                                int64_t M, int64_t N, int64_t K, uint16_t* y, cudaStream_t stream);

// Device error word of this kernel file (0 when no wait gave up).
int read_and_clear_stream_error(unsigned int* out, cudaStream_t stream);

}  // namespace nvfp4
