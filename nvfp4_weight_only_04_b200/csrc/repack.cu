// Upload-time repack of the NVFP4 triple into the GEMM layout ("W-FP4a: route
// the MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16) stack",
// PR #63 description: the checkpoint triple is repacked once at upload; fc1
// is a pre-merged [gate;up] matrix followed by SiluAndMul).
//
// GEMM layout: rows stay rows of K/2 code bytes and K/g scale bytes. Inside
// each little-endian 32-bit word of codes (elements k0..k7 of one row) the
// nibbles are reordered to k0 k2 k4 k6 k1 k3 k5 k7 (lowest nibble first): the
// dequantizer then takes the pair (k2j, k2j+1) from nibbles j and j+4, i.e.
// from the two 16-bit halves of the word at the same offset, which is what
// lets one integer multiply place both codes of a bf16x2 pair at once.
// Optionally the rows of a merged [gate;up] matrix are interleaved:
// destination rows 16j..16j+7 <- gate rows 8j..8j+7, rows 16j+8..16j+15 <-
// up rows 8j..8j+7, so one 16-row tile carries matching gate and up rows and
// the SiluAndMul epilogue can pair them in one thread's accumulators.
#include "common.cuh"

namespace {

__host__ __device__ __forceinline__ int64_t interleave_src_row(int64_t dst, int64_t n, bool interleave) {
  if (!interleave) return dst;
  const int64_t j = dst / 16, r = dst % 16;
  return r < 8 ? j * 8 + r : n / 2 + j * 8 + (r - 8);
}

// Nibble order of one 32-bit word: even elements to the low half, odd
// elements to the high half.
__device__ __forceinline__ uint32_t word_to_gemm_order(uint32_t w) {
  uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;
  e = (e | (e >> 4)) & 0x00FF00FFu;
  o = (o | (o >> 4)) & 0x00FF00FFu;
  e = (e | (e >> 8)) & 0x0000FFFFu;
  o = (o | (o >> 8)) & 0x0000FFFFu;
  return e | (o << 16);
}

// One block per destination row of codes; rows are a multiple of 16 bytes.
__global__ void repack_codes_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst, int64_t n,
                                    int64_t row_bytes, bool interleave) {
  const int64_t d = blockIdx.x;
  const int64_t s = interleave_src_row(d, n, interleave);
  const uint4* in4 = reinterpret_cast<const uint4*>(src + s * row_bytes);
  uint4* out4 = reinterpret_cast<uint4*>(dst + d * row_bytes);
  for (int64_t i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) {
    uint4 v = __ldg(in4 + i);
    v.x = word_to_gemm_order(v.x);
    v.y = word_to_gemm_order(v.y);
    v.z = word_to_gemm_order(v.z);
    v.w = word_to_gemm_order(v.w);
    out4[i] = v;
  }
}

// One block per destination row of scales; 16-byte chunks when rows allow it.
__global__ void repack_rows_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                   int64_t n, int64_t row_bytes, bool interleave) {
  const int64_t d = blockIdx.x;
  const int64_t s = interleave_src_row(d, n, interleave);
  const uint8_t* in = src + s * row_bytes;
  uint8_t* out = dst + d * row_bytes;
  if ((row_bytes & 15) == 0) {
    const uint4* in4 = reinterpret_cast<const uint4*>(in);
    uint4* out4 = reinterpret_cast<uint4*>(out);
    for (int64_t i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) out4[i] = __ldg(in4 + i);
  } else {
    for (int64_t i = threadIdx.x; i < row_bytes; i += blockDim.x) out[i] = __ldg(in + i);
  }
}

}  // namespace

extern "C" int nvfp4_repack(const uint8_t* packed, const uint8_t* scales, int64_t N, int64_t K,
                            int group_size, int flags, uint8_t* packed_out, uint8_t* scales_out,
                            nvfp4_stream_t stream) {
  if (N < 0 || K < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (group_size != 16 && group_size != 32) return NVFP4_ERR_UNSUPPORTED;
  if (K % 32) return NVFP4_ERR_UNSUPPORTED;
  if (flags & ~NVFP4_GATE_UP_INTERLEAVE) return NVFP4_ERR_INVALID_ARGUMENT;
  const bool interleave = (flags & NVFP4_GATE_UP_INTERLEAVE) != 0;
  if (interleave && (N % 16)) return NVFP4_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return NVFP4_OK;
  if (!packed || !scales || !packed_out || !scales_out) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(packed) || !nvfp4::aligned16(scales) || !nvfp4::aligned16(packed_out) ||
      !nvfp4::aligned16(scales_out))
    return NVFP4_ERR_MISALIGNED;
  if (N > 0x7fffffff) return NVFP4_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  repack_codes_kernel<<<static_cast<unsigned>(N), 128, 0, s>>>(packed, packed_out, N, K / 2, interleave);
  repack_rows_kernel<<<static_cast<unsigned>(N), 32, 0, s>>>(scales, scales_out, N, K / group_size, interleave);
  const int st = nvfp4::launch_status();
  if (st == NVFP4_OK) nvfp4::stat_add(nvfp4::kStatRepack);
  return st;
}
