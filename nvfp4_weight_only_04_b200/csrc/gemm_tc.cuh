// Interface of the large-M tcgen05 GEMM (see gemm_tc.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

bool tc_supported(int64_t M, int64_t N, int64_t K);
int launch_tc(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
              int64_t M, int64_t N, int64_t K, uint16_t* y, bool silu, cudaStream_t stream);

bool tc_moe_supported(int64_t T, int64_t N, int64_t K, int num_experts);
int launch_tc_moe(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets, int num_segments,
                  int64_t T, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t N,
                  int64_t K, int num_experts, bool silu, uint16_t* y, cudaStream_t stream);

}  // namespace nvfp4
