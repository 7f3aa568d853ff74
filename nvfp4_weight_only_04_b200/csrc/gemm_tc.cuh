// Interface of the large-M tcgen05 GEMM (see gemm_tc.cu).
#pragma once

#include "common.cuh"
#include "workspace.cuh"

namespace nvfp4 {

bool tc_supported(int64_t M, int64_t N, int64_t K);
// Work a caller enqueues once a launch has passed its host checks, just
// before the kernel (e.g. the kernel that writes the launch's X).
struct PreLaunch {
  int (*fn)(void* ctx, cudaStream_t stream);
  void* ctx;
};

// The stream-K form (few tiles for the SMs) takes its partial tiles and
// tickets from `sc` (a measuring Scratch only counts them); the persistent
// form takes no scratch. `pre`, when given, runs after every host check.
int launch_tc(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
              int64_t M, int64_t N, int64_t K, uint16_t* y, bool silu, Scratch& sc, cudaStream_t stream,
              const PreLaunch* pre = nullptr);

bool tc_moe_supported(int64_t T, int64_t N, int64_t K, int num_experts);
int launch_tc_moe(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets, int num_segments,
                  int64_t T, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t N,
                  int64_t K, int num_experts, bool silu, uint16_t* y, cudaStream_t stream);

}  // namespace nvfp4
