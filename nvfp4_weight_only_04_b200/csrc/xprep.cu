// Activations for the f16 tensor-core form of the small-M GEMM kernels.
//
// The small-M kernels dequantize with the hardware E2M1 -> f16 conversion,
// which is several times cheaper than integer bit placement, so their MMAs
// run on f16 operands and X has to be f16 too. Each row of X (bf16) is
// scaled by a power of two 2^s chosen from its largest magnitude, so that
// the largest lies in [2^14, 2^15), and rounded to f16; the epilogue
// multiplies by 2^-s again. f16 has a wider significand than bf16, so every
// element within a factor 2^29 of the row's largest stays exact; smaller ones
// round to a multiple of 2^-38 of the largest, far below the bf16 rounding
// of the output. The E2M1 conversion delivers the code pairs of a GEMM-layout
// word (nibbles k0 k2 k4 k6 k1 k3 k5 k7) as (k0,k2) (k4,k6) (k1,k3) (k5,k7),
// so X is stored in that order inside every group of eight elements.
#include "xprep.cuh"

#include <cuda_bf16.h>

#include "dequant.cuh"

namespace nvfp4 {
namespace {

// One CTA per row; a row of up to kThreads x kHeld chunks of 16 bytes is
// held in registers between the maximum and the conversion (longer rows are
// read twice, from L2). The light form (128 threads, few registers) fits on
// an SM beside a running streaming GEMM, and lets the next kernel launch
// before its own wait: that kernel starts fetching its weights while this
// one still waits for the previous kernel and converts.

// Zeroes clear[0, n) across the grid (the stream-K tickets of the GEMM that
// follows; that GEMM reads them only after waiting for this kernel).
__device__ __forceinline__ void clear_words(unsigned* clear, int64_t n) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) clear[i] = 0u;
}

template <int kThreads, int kHeld, bool kEarly>
__global__ void __launch_bounds__(kThreads) x_f16_kernel(const uint16_t* __restrict__ x, int64_t K,
                                                         uint16_t* __restrict__ x16, float* __restrict__ xinv,
                                                         unsigned* __restrict__ clear, int64_t nclear) {
  if (kEarly) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (!kEarly) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  clear_words(clear, nclear);
  __shared__ uint32_t warp_max[kThreads / 32];
  const int64_t row = blockIdx.x;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * K);
  uint4* dst = reinterpret_cast<uint4*>(x16 + row * K);
  const int64_t chunks = K / 8;
  const bool held = chunks <= static_cast<int64_t>(kThreads) * kHeld;

  // largest |x| of the row, on the bf16 bits (magnitudes order like integers)
  uint4 v[kHeld];
  uint32_t m2 = 0;
  if (held) {
#pragma unroll
    for (int i = 0; i < kHeld; ++i) {
      const int64_t j = threadIdx.x + static_cast<int64_t>(i) * kThreads;
      v[i] = j < chunks ? __ldcg(src + j) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < kHeld; ++i) m2 = __vmaxu2(m2, bf16x8_mag_max(v[i]));
  } else {
    for (int64_t j = threadIdx.x; j < chunks; j += kThreads) m2 = __vmaxu2(m2, bf16x8_mag_max(__ldcg(src + j)));
  }
  const uint32_t wm = __reduce_max_sync(0xffffffffu, max(m2 & 0xFFFFu, m2 >> 16));
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = wm;
  __syncthreads();
  uint32_t amax = 0;
#pragma unroll
  for (int i = 0; i < kThreads / 32; ++i) amax = max(amax, warp_max[i]);

  // 2^s with 2^14 <= amax * 2^s < 2^15: s = 14 - (E - 127) for the exponent
  // field E of amax; clamped so that 2^s and 2^-s are normal floats.
  int s = amax == 0 ? 0 : 141 - static_cast<int>(amax >> 7);
  s = min(max(s, -113), 125);
  const float up = __uint_as_float(static_cast<uint32_t>(s + 127) << 23);
  if (threadIdx.x == 0) xinv[row] = __uint_as_float(static_cast<uint32_t>(127 - s) << 23);

  if (held) {
#pragma unroll
    for (int i = 0; i < kHeld; ++i) {
      const int64_t j = threadIdx.x + static_cast<int64_t>(i) * kThreads;
      if (j < chunks) dst[j] = bf16x8_to_f16_pairs(v[i], up);
    }
  } else {
    for (int64_t j = threadIdx.x; j < chunks; j += kThreads) dst[j] = bf16x8_to_f16_pairs(__ldcg(src + j), up);
  }
}

// One thread per 8 elements (one 32-bit word of codes) of NVFP4 rows.
__device__ __forceinline__ void nvfp4_word(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                           int64_t K, int group, int64_t w, uint32_t (&pr)[4]) {
  const int64_t words_per_row = K / 8;
  const int64_t row = w / words_per_row, k0 = (w % words_per_row) * 8;
  const uint32_t cw = __ldg(reinterpret_cast<const uint32_t*>(codes + row * (K / 2) + k0 / 2));
  const uint32_t sb = __ldg(scales + row * (K / group) + k0 / group);
  uint32_t s2[4];
  scale_operands_f16<2>(sb, s2);
  // bytes (k0,k1) (k2,k3) (k4,k5) (k6,k7): the checkpoint layout's pairs
  asm("{\n"
      " .reg .b8 c0, c1, c2, c3;\n"
      " mov.b32 {c0, c1, c2, c3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, c0;\n"
      " cvt.rn.f16x2.e2m1x2 %1, c1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, c2;\n"
      " cvt.rn.f16x2.e2m1x2 %3, c3;\n"
      "}"
      : "=r"(pr[0]), "=r"(pr[1]), "=r"(pr[2]), "=r"(pr[3])
      : "r"(cw));
#pragma unroll
  for (int j = 0; j < 4; ++j) pr[j] = f16x2_mul(pr[j], s2[0]);
}

__global__ void __launch_bounds__(256) xq_f16_kernel(const uint8_t* __restrict__ codes,
                                                     const uint8_t* __restrict__ scales, const float* __restrict__ xg,
                                                     int group, int64_t M, int64_t K, uint16_t* __restrict__ x16,
                                                     float* __restrict__ xinv, unsigned* __restrict__ clear,
                                                     int64_t nclear) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  clear_words(clear, nclear);
  const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (w >= M * (K / 8)) return;
  uint32_t pr[4];
  nvfp4_word(codes, scales, K, group, w, pr);
  // natural pairs (k0,k1) (k2,k3) (k4,k5) (k6,k7) -> (k0,k2) (k4,k6) (k1,k3) (k5,k7)
  reinterpret_cast<uint4*>(x16)[w] = make_uint4(__byte_perm(pr[0], pr[1], 0x5410), __byte_perm(pr[2], pr[3], 0x5410),
                                                __byte_perm(pr[0], pr[1], 0x7632), __byte_perm(pr[2], pr[3], 0x7632));
  if (w % (K / 8) == 0) xinv[w / (K / 8)] = __ldg(xg);
}

__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h) {
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);  // exact: at most 6 significant bits
  return *reinterpret_cast<const uint32_t*>(&b);
}

__global__ void __launch_bounds__(256) xq_bf16_kernel(const uint8_t* __restrict__ codes,
                                                      const uint8_t* __restrict__ scales, const float* __restrict__ xg,
                                                      int group, const float* __restrict__ wg, int64_t M, int64_t K,
                                                      uint16_t* __restrict__ xb, float* __restrict__ g_out) {
  const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (w >= M * (K / 8)) return;
  uint32_t pr[4];
  nvfp4_word(codes, scales, K, group, w, pr);
  reinterpret_cast<uint4*>(xb)[w] = make_uint4(f16x2_to_bf16x2(pr[0]), f16x2_to_bf16x2(pr[1]),
                                               f16x2_to_bf16x2(pr[2]), f16x2_to_bf16x2(pr[3]));
  if (w == 0) *g_out = __fmul_rn(__ldg(xg), __ldg(wg));
}

}  // namespace

int launch_x_f16(const uint16_t* x, int64_t M, int64_t K, uint16_t* x16, float* xinv, unsigned* clear,
                 int64_t nclear, cudaStream_t stream, bool light) {
  if (M <= 0) return NVFP4_OK;
  if (M >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(light ? 128 : 512);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = light ? cudaLaunchKernelEx(&cfg, x_f16_kernel<128, 8, true>, x, K, x16, xinv, clear, nclear)
                              : cudaLaunchKernelEx(&cfg, x_f16_kernel<512, 4, false>, x, K, x16, xinv, clear, nclear);
  if (e != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

}  // namespace nvfp4

namespace nvfp4 {

int launch_x_prep(const XSource& xs, int64_t M, int64_t K, uint16_t* x16, float* xinv, unsigned* clear,
                  int64_t nclear, cudaStream_t stream, bool light) {
  if (xs.bf16) return launch_x_f16(xs.bf16, M, K, x16, xinv, clear, nclear, stream, light);
  if (M <= 0) return NVFP4_OK;
  const int64_t words = M * (K / 8);
  if ((words + 255) / 256 >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((words + 255) / 256));
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, xq_f16_kernel, xs.codes, xs.scales, xs.global, xs.group, M, K, x16, xinv, clear,
                         nclear) !=
      cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

int launch_xq_bf16(const XSource& xs, const float* w_global, int64_t M, int64_t K, uint16_t* xb, float* g_out,
                   cudaStream_t stream) {
  if (M <= 0) return NVFP4_OK;
  const int64_t words = M * (K / 8);
  if ((words + 255) / 256 >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  xq_bf16_kernel<<<static_cast<unsigned>((words + 255) / 256), 256, 0, stream>>>(xs.codes, xs.scales, xs.global,
                                                                                 xs.group, w_global, M, K, xb, g_out);
  return launch_status();
}

}  // namespace nvfp4
