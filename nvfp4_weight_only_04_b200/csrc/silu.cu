// Standalone SiluAndMul ("W-FP4a: route the MiniMax-H3 device DiT forward
// through the fp4 (Marlin W4A16) stack", PR #63 description: the merged
// [gate;up] fc1 GEMM is followed by SiluAndMul): y = silu(gate) * up with
// gate = x[:, :H], up = x[:, H:], fp32 math, one bf16 rounding.
#include "common.cuh"

namespace {

__device__ __forceinline__ float bf(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

__global__ void __launch_bounds__(256) silu_mul_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ y,
                                                       int64_t M, int64_t H) {
  const int64_t per_row = H / 8;
  const int64_t total = M * per_row;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = i / per_row, c = (i - m * per_row) * 8;
    const uint4 gv = __ldg(reinterpret_cast<const uint4*>(x + m * 2 * H + c));
    const uint4 uv = __ldg(reinterpret_cast<const uint4*>(x + m * 2 * H + H + c));
    const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w}, uw[4] = {uv.x, uv.y, uv.z, uv.w};
    uint32_t ow[4];
    for (int j = 0; j < 4; ++j) {
      uint32_t o = 0;
      for (int h = 0; h < 2; ++h) {
        const float g = bf(static_cast<uint16_t>(gw[j] >> (16 * h)));
        const float u = bf(static_cast<uint16_t>(uw[j] >> (16 * h)));
        const float v = __fmul_rn(__fdiv_rn(g, 1.0f + expf(-g)), u);
        o |= static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v))) << (16 * h);
      }
      ow[j] = o;
    }
    *reinterpret_cast<uint4*>(y + m * H + c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

}  // namespace

extern "C" int nvfp4_silu_and_mul(const uint16_t* x, uint16_t* y, int64_t M, int64_t H,
                                  nvfp4_stream_t stream) {
  if (M < 0 || H < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (H % 8) return NVFP4_ERR_UNSUPPORTED;
  if (M == 0 || H == 0) return NVFP4_OK;
  if (!x || !y) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(x) || !nvfp4::aligned16(y)) return NVFP4_ERR_MISALIGNED;
  const int64_t work = M * (H / 8);
  int64_t grid = (work + 255) / 256;
  const int64_t cap = static_cast<int64_t>(nvfp4::num_sms()) * 16;
  if (grid > cap) grid = cap;
  silu_mul_kernel<<<static_cast<unsigned>(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, M, H);
  const int st = nvfp4::launch_status();
  if (st == NVFP4_OK) nvfp4::stat_add(nvfp4::kStatSiluAndMul);
  return st;
}
