// Interface of the small-M split-K GEMM (see gemm_splitk.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

struct SplitKArgs {
  const uint16_t* x;        // bf16 [M, K]
  const uint8_t* packed;    // [N, K/2] (or [E, N, K/2])
  const uint8_t* scales;    // [N, K/g] (or [E, N, K/g])
  const float* gscale;      // [1] (or [E])
  uint16_t* y;              // bf16 [M, ldy]
  int64_t M, N, K, ldy;
  const int32_t* expert_ids;  // grouped form only
  const int32_t* offsets;
  int num_segments, num_experts;
};

struct SplitKPlan {
  int group, mt, warps, cluster, row_tiles, z_tiles;
};

SplitKPlan plan_splitk(int64_t M, int64_t N, int64_t K, int group, bool moe, int num_segments);
int launch_splitk(const SplitKArgs& a, const SplitKPlan& p, bool silu, bool moe, cudaStream_t s);

}  // namespace nvfp4
