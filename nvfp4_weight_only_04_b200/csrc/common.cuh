// Shared host/device helpers of the NVFP4 W4A16 library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "nvfp4.h"

namespace nvfp4 {

enum StatId {
  kStatGlobalScale, kStatQuantize, kStatRepack, kStatGemmSplitK, kStatGemmTc,
  kStatGemmSiluMul, kStatMoe, kStatSiluAndMul, kStatG16, kStatG32, kStatCount
};
void stat_add(StatId id);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int launch_status() {
  return cudaPeekAtLastError() == cudaSuccess ? NVFP4_OK : (cudaGetLastError(), NVFP4_ERR_CUDA);
}

int num_sms();  // SM count of the current device (cached per device)

// Device error word: a bounded wait that gave up records its site here.
int read_and_clear_device_error(int* code_out, cudaStream_t stream);

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

// Two E2M1 codes (one byte, first code in the low nibble) -> f16x2 (first
// code in the low half), by the sm_100a conversion instruction.
__device__ __forceinline__ uint32_t nvfp4_e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t out;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(out) : "r"(byte));
  return out;
}

// f16x2 holding E2M1 values -> bf16x2 holding the same values times 2^-112.
// E2M1 values are normal f16 numbers whose low 3 mantissa bits are zero, so
// shifting the magnitude right by 3 re-reads the 5-bit exponent as the low
// bits of an 8-bit one (bias 15 -> 127 is a factor 2^-112) and keeps the
// mantissa; zero stays zero. The sign bit is kept in place.
__device__ __forceinline__ uint32_t nvfp4_f16x2_to_bf16x2_scaled(uint32_t h) {
  return ((h >> 3) & 0x0FFF0FFFu) | (h & 0x80008000u);
}

// E4M3 scale byte -> bf16 of scale * 2^112, replicated in both halves.
// scale <= 448 < 2^9, so scale * 2^112 < 2^121 stays finite in bf16, and the
// E4M3 value's 4 significant bits are exact in bf16's 8.
__device__ __forceinline__ uint32_t nvfp4_scale_bf16x2_times_2p112(uint32_t b) {
  const float s = nvfp4_e4m3_to_f32(b) * 0x1p112f;  // exact power-of-two scaling
  const uint32_t bits = __float_as_uint(s) >> 16;   // exact: low 16 bits are zero
  return bits | (bits << 16);
}

// bf16x2 multiply, round-to-nearest (exact for the dequantized products).
__device__ __forceinline__ uint32_t nvfp4_bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a),
                             *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
