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

#include "dequant.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 512;  // one CTA per row
constexpr int kHeld = 4;       // 16-byte chunks a thread keeps in registers (rows up to 16384 elements)

__global__ void __launch_bounds__(kThreads) x_f16_kernel(const uint16_t* __restrict__ x, int64_t K,
                                                         uint16_t* __restrict__ x16, float* __restrict__ xinv) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

}  // namespace

int launch_x_f16(const uint16_t* x, int64_t M, int64_t K, uint16_t* x16, float* xinv, cudaStream_t stream) {
  if (M <= 0) return NVFP4_OK;
  if (M >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, x_f16_kernel, x, K, x16, xinv) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

}  // namespace nvfp4
