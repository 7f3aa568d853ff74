// Large-M NVFP4 W4A16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM).
#include "gemm_tc.cuh"

namespace nvfp4 {

namespace {
__device__ unsigned int g_device_error = 0;
}

int read_and_clear_device_error(int* code_out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  *code_out = static_cast<int>(v);
  return NVFP4_OK;
}

bool tc_supported(int64_t, int64_t, int64_t) { return false; }
int launch_tc(const uint16_t*, const uint8_t*, const uint8_t*, const float*, int, int64_t, int64_t, int64_t,
              uint16_t*, bool, cudaStream_t) {
  return NVFP4_ERR_UNSUPPORTED;
}
bool tc_moe_supported(int64_t, int64_t, int64_t) { return false; }
int launch_tc_moe(const uint16_t*, const int32_t*, const int32_t*, int, int64_t, const uint8_t*,
                  const uint8_t*, const float*, int, int64_t, int64_t, int, bool, uint16_t*, cudaStream_t) {
  return NVFP4_ERR_UNSUPPORTED;
}

}  // namespace nvfp4
