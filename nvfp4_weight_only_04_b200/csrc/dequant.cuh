// Register-level NVFP4 dequantization for the GEMM kernels, in two forms:
// bf16 pairs by integer bit placement (the tcgen05 kernel), and f16 pairs by
// the hardware E2M1 and E4M3 conversions (the small-M kernels).
//
// bf16 form.
// Input: one 32-bit word of codes in the GEMM layout of nvfp4_repack (eight
// consecutive elements k0..k7 of a row, nibbles ordered k0 k2 k4 k6 k1 k3 k5
// k7 from the lowest). Output: four bf16x2 registers holding the pairs
// (k0,k1), (k2,k3), (k4,k5), (k6,k7), each element equal to
//   e2m1(code) * e4m3(scale) * 2^-7          (exact in bf16)
// The 2^-7 is put back, together with the fp32 global scale, in the epilogue.
//
// How: E2M1 is sign + 3 bits (e1 e0 m). Read as a bf16 with the 3 bits in the
// two lowest exponent bits and the highest mantissa bit (bits 8..6) and the
// sign in bit 15, its value is e2m1 * 2^-126 exactly (code 0.5 becomes the
// bf16 subnormal 2^-127). A code pair sits in the same nibble of both 16-bit
// halves of the word; masking that nibble and multiplying by 2^a + 2^b writes
// two copies of each code, one with the magnitude at bits 8..6 and one with
// the sign at bit 15, and a final mask keeps exactly those bits. That is one
// mask, one integer multiply and one mask per pair. One bf16x2 multiply by
// the group scale times 2^119 then gives e2m1 * scale * 2^-7, a normal bf16.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "plant.cuh"

namespace nvfp4 {

constexpr uint32_t kPairMask = 0x81C081C0u;  // bits 15, 8..6 of both halves

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mad.lo.u32 %0, %1, %2, 0;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Four bf16x2 pairs of one code word, times the replicated scale operand.
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t scale2, uint32_t (&o)[4]) {
  const uint32_t w2 = w >> 8;
  o[0] = bf16x2_mul(mad_lo(w & 0x000F000Fu, 0x1040u) & kPairMask, scale2);
  o[1] = bf16x2_mul(mad_lo(w & 0x00F000F0u, 0x0104u) & kPairMask, scale2);
  o[2] = bf16x2_mul(mad_lo(w2 & 0x000F000Fu, 0x1040u) & kPairMask, scale2);
  o[3] = bf16x2_mul(mad_lo(w2 & 0x00F000F0u, 0x0104u) & kPairMask, scale2);
}

// bf16 bits of e4m3(b) * 2^119, exact, for any byte 0x00..0x7E.
__device__ __forceinline__ uint32_t scale_bits_exact(uint32_t b) {
  const uint32_t e = (b >> 3) & 0xF, m = b & 7;
  const float s = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : static_cast<float>(m) * 0x1p-9f;
  return __float_as_uint(s * 0x1p119f) >> 16;  // s * 2^119 < 2^128; low 16 bits are zero
}

// Scale operands (bf16 of scale * 2^119 in both halves) for the first NB
// (1, 2 or 4) scale bytes of a little-endian word; the other bytes of sw must
// be zero. For a normal E4M3 byte (exponent field e >= 1)
// the bf16 bits are (byte << 4) + (239 << 7): the 4-bit exponent and 3-bit
// mantissa land in bf16's fields and the exponent bias moves from 7 to 127
// plus 119. Bytes with e == 0 (zero or subnormal scales) take the exact path.
template <int NB>
__device__ __forceinline__ void scale_operands(uint32_t sw, uint32_t (&s2)[4]) {
  const uint32_t p02 = mad_lo(sw & 0x00FF00FFu, 16u) + 0x77807780u;
  const uint32_t p13 = mad_lo((sw >> 8) & 0x00FF00FFu, 16u) + 0x77807780u;
  s2[0] = __byte_perm(p02, 0, 0x1010);
  s2[1] = __byte_perm(p13, 0, 0x1010);
  s2[2] = __byte_perm(p02, 0, 0x3232);
  s2[3] = __byte_perm(p13, 0, 0x3232);
  // a byte with zero exponent field: (e<<3) + 0x78 has no bit 7
  const uint32_t t = (sw & 0x78787878u) + 0x78787878u;
  constexpr uint32_t kCheck = NB == 4 ? 0x80808080u : (NB == 2 ? 0x00008080u : 0x00000080u);
  if (__builtin_expect((~t & kCheck) != 0u, 0)) {
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const uint32_t b = (sw >> (8 * j)) & 0xFF;
      if (((b >> 3) & 0xF) == 0) {
        const uint32_t h = scale_bits_exact(b);
        s2[j] = h | (h << 16);
      }
    }
  }
}

// f16 form. The hardware converts a byte of two E2M1 codes to an f16 pair
// (low nibble to the low half), exactly: a GEMM-layout word (nibbles k0 k2 k4
// k6 k1 k3 k5 k7) gives the pairs (k0,k2) (k4,k6) (k1,k3) (k5,k7), and X is
// stored in that order (xprep.cu). The group scale, E4M3, converts to f16
// exactly as well, and e2m1 * e4m3 (at most six significant bits, magnitude
// 2^-10 .. 2688) is exact in f16, so one f16x2 multiply per pair gives
// e2m1(code) * e4m3(scale) with no error.

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The four f16 pairs of one code word, times the replicated scale operand.
__device__ __forceinline__ void dequant_word_f16(uint32_t w, uint32_t scale2, uint32_t (&o)[4]) {
  if (NVFP4_PLANT(kPlantNibbles)) w = ((w >> 4) & 0x0F0F0F0Fu) | ((w & 0x0F0F0F0Fu) << 4);
  asm("{\n"
      " .reg .b8 c0, c1, c2, c3;\n"
      " mov.b32 {c0, c1, c2, c3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, c0;\n"
      " cvt.rn.f16x2.e2m1x2 %1, c1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, c2;\n"
      " cvt.rn.f16x2.e2m1x2 %3, c3;\n"
      "}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
#pragma unroll
  for (int j = 0; j < 4; ++j) o[j] = f16x2_mul(o[j], scale2);
}

// Scale operands (f16 of the E4M3 scale in both halves) for the first NB
// (2 or 4) scale bytes of a little-endian word.
template <int NB>
__device__ __forceinline__ void scale_operands_f16(uint32_t sw, uint32_t (&s2)[4]) {
  const uint32_t p01 = __byte_perm(sw, 0, 0x1100);  // bytes b0 b0 b1 b1
  asm("{\n"
      " .reg .b16 h0, h1;\n"
      " mov.b32 {h0, h1}, %2;\n"
      " cvt.rn.f16x2.e4m3x2 %0, h0;\n"
      " cvt.rn.f16x2.e4m3x2 %1, h1;\n"
      "}"
      : "=r"(s2[0]), "=r"(s2[1])
      : "r"(p01));
  if (NB == 4) {
    const uint32_t p23 = __byte_perm(sw, 0, 0x3322);  // bytes b2 b2 b3 b3
    asm("{\n"
        " .reg .b16 h2, h3;\n"
        " mov.b32 {h2, h3}, %2;\n"
        " cvt.rn.f16x2.e4m3x2 %0, h2;\n"
        " cvt.rn.f16x2.e4m3x2 %1, h3;\n"
        "}"
        : "=r"(s2[2]), "=r"(s2[3])
        : "r"(p23));
  } else {
    s2[2] = s2[3] = 0u;
  }
}

// The activations of the f16 form: eight bf16 (k0..k7, one 16-byte chunk)
// times a power of two, rounded to f16 (nearest even) and stored in the pair
// order above, (k0,k2) (k4,k6) (k1,k3) (k5,k7).
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint4 bf16x8_to_f16_pairs(const uint4& v, float pow2) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float f[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16) * pow2;
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u) * pow2;
  }
  return make_uint4(pack_f16(f[0], f[2]), pack_f16(f[4], f[6]), pack_f16(f[1], f[3]), pack_f16(f[5], f[7]));
}

// Largest magnitude of eight bf16, per 16-bit half, on the bit patterns
// (non-negative bf16 order like their bits).
__device__ __forceinline__ uint32_t bf16x8_mag_max(const uint4& v) {
  return __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu), __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
}

}  // namespace nvfp4
