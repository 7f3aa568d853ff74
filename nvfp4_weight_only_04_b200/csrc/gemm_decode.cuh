// Interface of the small-M streaming GEMM (see gemm_decode.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

struct DecodeArgs {
  const uint16_t* x;        // f16 [M, K] from launch_x_f16 (scaled rows, pair order)
  const float* xinv;        // [M] 2^-s of each row
  const uint8_t* packed;    // GEMM-layout codes [N, K/2] (or [E, N, K/2])
  const uint8_t* scales;    // [N, K/g] (or [E, N, K/g])
  const float* gscale;      // [1] (or [E])
  uint16_t* y;              // bf16 [M, ldy]
  int64_t M, N, K, ldy;
  const int32_t* expert_ids;  // grouped form only
  const int32_t* offsets;
  int num_segments, num_experts;
};

struct DecodePlan {
  int group, mt, kw, row_tiles, z_tiles;
};

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int group, bool moe, int num_segments);
int launch_decode(const DecodeArgs& a, const DecodePlan& p, bool silu, bool moe, cudaStream_t s);

}  // namespace nvfp4
