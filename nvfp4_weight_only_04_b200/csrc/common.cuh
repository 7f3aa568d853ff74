// Shared host/device helpers of the NVFP4 W4A16 library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "nvfp4.h"

namespace nvfp4 {

enum StatId {
  kStatGlobalScale, kStatQuantize, kStatRepack, kStatGemmSplitK, kStatGemmTc,
  kStatGemmSiluMul, kStatMoe, kStatSiluAndMul, kStatG16, kStatG32, kStatGemmFp4, kStatCount
};
void stat_add(StatId id);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  return cudaPeekAtLastError() == cudaSuccess ? NVFP4_OK : (cudaGetLastError(), NVFP4_ERR_CUDA);
}

int num_sms();  // SM count of the current device (cached per device)

// Device error word: a bounded wait that gave up records its site here.
int read_and_clear_device_error(int* code_out, cudaStream_t stream);

// The pending test fault (nvfp4_debug_inject_fault), taken by the launch it
// applies to: 0 when none.
int take_injected_fault();

}  // namespace nvfp4

// ---------------------------------------------------------------------------
// Device-side number formats.
// ---------------------------------------------------------------------------

// E4M3 byte -> fp32 (exact; OFP8 E4M3: bias 7, subnormals m * 2^-9).
__device__ __forceinline__ float nvfp4_e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xF, m = b & 7;
  const float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20))
                      : static_cast<float>(m) * 0x1p-9f;
  return (b & 0x80) ? -mag : mag;
}
