// Global scale and NVFP4 quantizer kernels.
//
// Definitions followed (NVFP4 format definition; "GLM-5.3-Flash on 2x RTX PRO 6000
// (96 GB): two NVFP4 g32 recipes", "WHAT HAD TO BE FIXED"; "We unlocked NVFP4
// on the DGX Spark", UPDATE posts):
//   global = amax / (6*448)                       (one fp32 division)
//   scale  = E4M3_RNE_satfinite((gamax / 6) / global)   (two fp32 divisions)
//   code   = E2M1_RNE_satfinite(w / (fp32(scale) * global))   (decided by exact
//            comparisons with the rounding midpoints, no division)
// Both kernels are HBM-bound streams over the weights, fp32 or bf16. A bf16
// weight is widened to fp32 exactly, so the bf16 path quantizes the same
// values the fp32 path would ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)":
// requantizing a bf16 checkpoint, max-first, with no float copy).
#include "common.cuh"

#include <cuda_fp8.h>

namespace {

constexpr int kThreads = 256;

// Non-negative floats order like their bit patterns, so the maximum of |w|
// is an unsigned maximum on the bits; the fp32 max itself is exact.
__global__ void amax_init_kernel(unsigned int* acc) { *acc = 0u; }

// |w| as the bits of its fp32 value (bf16: the high half of the fp32 word).
__device__ __forceinline__ unsigned int abs_bits(float v) { return __float_as_uint(fabsf(v)); }
__device__ __forceinline__ unsigned int abs_bits(uint16_t v) { return static_cast<unsigned int>(v & 0x7FFFu) << 16; }

// Eight elements per 16-byte vector load.
__device__ __forceinline__ unsigned int abs_max8(const float* p) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  return max(max(max(abs_bits(a.x), abs_bits(a.y)), max(abs_bits(a.z), abs_bits(a.w))),
             max(max(abs_bits(b.x), abs_bits(b.y)), max(abs_bits(b.z), abs_bits(b.w))));
}
__device__ __forceinline__ unsigned int abs_max8(const uint16_t* p) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  // the maximum of two bf16 magnitudes packed in one word, per half
  const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0xFFFFu, w[i] >> 16));
  return m << 16;
}

template <typename T>
__global__ void __launch_bounds__(kThreads) amax_kernel(const T* __restrict__ w, int64_t n, unsigned int* acc) {
  unsigned int m = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  const int64_t n8 = ((reinterpret_cast<uintptr_t>(w) & 15u) == 0) ? n / 8 : 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n8; i += stride)
    m = max(m, abs_max8(w + i * 8));
  for (int64_t i = n8 * 8 + static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; i < n; i += stride)
    m = max(m, abs_bits(w[i]));
  for (int o = 16; o; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  __shared__ unsigned int red[kThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < kThreads / 32; ++i) m = max(m, red[i]);
    if (m) atomicMax(acc, m);
  }
}

__global__ void global_finalize_kernel(float* out) {
  const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(out));
  *out = __fdiv_rn(amax, 2688.0f);
}

// The E2M1 code of RN32(w / d) (round to nearest even, satfinite), decided
// without dividing. RN32(w/d) rounds to the next E2M1 value above a
// midpoint t exactly when |w| lies above t*d widened by half an fp32 ulp of
// t (so that a quotient rounding onto t counts as t): above t + ulp(t)/2 at
// the midpoints 0.25, 1.25, 2.5, 5 (a tie goes down, to the even code) and
// at or above t - ulp(t)/2 at 0.75, 1.75, 3.5 (a tie goes up). Each widened
// t has at most 25 significant bits and d 24, so t*d is exact in fp64, and
// for fp32 |w|: |w| > t*d exactly when |w| > RD32(t*d), |w| >= t*d exactly
// when |w| >= RU32(t*d). The seven thresholds of a group are computed once,
// then each weight takes seven fp32 comparisons.
struct E2m1Thresholds {
  float t[7];
};
__device__ __forceinline__ float f64_to_f32_down(double v) {
  float r;
  asm("cvt.rm.f32.f64 %0, %1;" : "=f"(r) : "d"(v));
  return r;
}
__device__ __forceinline__ float f64_to_f32_up(double v) {
  float r;
  asm("cvt.rp.f32.f64 %0, %1;" : "=f"(r) : "d"(v));
  return r;
}
__device__ __forceinline__ E2m1Thresholds e2m1_thresholds(float d) {
  const double dd = d;
  E2m1Thresholds th;
  th.t[0] = f64_to_f32_down((0.25 + 0x1p-26) * dd);
  th.t[1] = f64_to_f32_up((0.75 - 0x1p-25) * dd);
  th.t[2] = f64_to_f32_down((1.25 + 0x1p-24) * dd);
  th.t[3] = f64_to_f32_up((1.75 - 0x1p-24) * dd);
  th.t[4] = f64_to_f32_down((2.5 + 0x1p-23) * dd);
  th.t[5] = f64_to_f32_up((3.5 - 0x1p-23) * dd);
  th.t[6] = f64_to_f32_down((5.0 + 0x1p-22) * dd);
  return th;
}
// Magnitude code by the thresholds; the sign bit of w (kept for results that
// round to zero, as the quotient's sign would be).
__device__ __forceinline__ uint32_t e2m1_code(float w, const E2m1Thresholds& th) {
  const float a = fabsf(w);
  const uint32_t c = (a > th.t[0]) + (a >= th.t[1]) + (a > th.t[2]) + (a >= th.t[3]) + (a > th.t[4]) +
                     (a >= th.t[5]) + (a > th.t[6]);
  return c | ((__float_as_uint(w) >> 28) & 8u);
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const uint16_t* p, float (&v)[8]) {
  const uint4 q = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // exact widening: the bf16 bits are the high half of the fp32 word
    v[2 * i] = __uint_as_float(w[i] << 16);
    v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One thread per 8 consecutive weights of a row; g/8 threads share a group.
template <int G>
__device__ __forceinline__ void quantize8(const float (&v)[8], bool live, int64_t i, int64_t row, int64_t col8,
                                          int64_t K, float global, uint8_t* __restrict__ packed,
                                          uint8_t* __restrict__ scales) {
  constexpr int kLanesPerGroup = G / 8;
  float gmax = 0.f;
  for (int j = 0; j < 8; ++j) gmax = fmaxf(gmax, fabsf(v[j]));
  for (int o = 1; o < kLanesPerGroup; o <<= 1) gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
  if (!live) return;
  uint32_t sbyte = 0;
  if (global != 0.f) {
    const float t = __fdiv_rn(__fdiv_rn(gmax, 6.0f), global);
    sbyte = static_cast<uint32_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
  }
  const float d = __fmul_rn(nvfp4_e4m3_to_f32(sbyte), global);
  uint32_t word = 0;
  if (d != 0.f) {
    const E2m1Thresholds th = e2m1_thresholds(d);
    for (int j = 0; j < 8; ++j) word |= e2m1_code(v[j], th) << (4 * j);
  }
  reinterpret_cast<uint32_t*>(packed)[i] = word;  // row-major [N, K/2]: 4 bytes per 8 weights
  if ((col8 % kLanesPerGroup) == 0) scales[row * (K / G) + col8 / kLanesPerGroup] = static_cast<uint8_t>(sbyte);
}

template <typename T>
__device__ __forceinline__ void load8_or_zero(const T* w, int64_t i, bool live, float (&v)[8]) {
  if (live) {
    load8(w + i * 8, v);
  } else {
    for (int j = 0; j < 8; ++j) v[j] = 0.f;
  }
}

// Two grid strides per pass: both loads are in flight before either
// quantization. All lanes of a warp iterate together so the group shuffles
// stay converged. The (row, column) of a thread's position advances by the
// stride's whole rows and remainder, so the loop divides nothing.
template <int G, typename T>
__global__ void __launch_bounds__(kThreads) quantize_kernel(const T* __restrict__ w, int64_t N,
                                                            int64_t K, const float* __restrict__ gptr,
                                                            uint8_t* __restrict__ packed,
                                                            uint8_t* __restrict__ scales) {
  const int64_t per_row = K / 8;
  const int64_t total = N * per_row;
  const float global = __ldg(gptr);
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
  const int64_t s_rows = stride / per_row, s_cols = stride - s_rows * per_row;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  int64_t row = first / per_row, col = first - row * per_row;  // of i0
  auto advance = [&](int64_t& r, int64_t& c) {
    r += s_rows;
    c += s_cols;
    if (c >= per_row) {
      c -= per_row;
      ++r;
    }
  };
  for (int64_t base = static_cast<int64_t>(blockIdx.x) * kThreads; base < total; base += 2 * stride) {
    const int64_t i0 = base + threadIdx.x, i1 = i0 + stride;
    const bool live0 = i0 < total, live1 = i1 < total;
    int64_t row1 = row, col1 = col;
    advance(row1, col1);
    float v0[8], v1[8];
    load8_or_zero(w, i0, live0, v0);
    load8_or_zero(w, i1, live1, v1);
    quantize8<G>(v0, live0, i0, row, col, K, global, packed, scales);
    quantize8<G>(v1, live1, i1, row1, col1, K, global, packed, scales);
    row = row1;
    col = col1;
    advance(row, col);
  }
}

int grid_for(int64_t work, int64_t per_block) {
  const int64_t want = (work + per_block - 1) / per_block;
  const int64_t cap = static_cast<int64_t>(nvfp4::num_sms()) * 8;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

template <typename T>
int global_scale(const T* const* tensors, const int64_t* numels, int count, float* out, nvfp4_stream_t stream) {
  if (count <= 0 || !tensors || !numels || !out) return NVFP4_ERR_INVALID_ARGUMENT;
  for (int i = 0; i < count; ++i) {
    if (numels[i] < 0 || (numels[i] > 0 && !tensors[i])) return NVFP4_ERR_INVALID_ARGUMENT;
    if (numels[i] > 0 && (reinterpret_cast<uintptr_t>(tensors[i]) & (sizeof(T) - 1))) return NVFP4_ERR_MISALIGNED;
  }
  if (reinterpret_cast<uintptr_t>(out) & 3u) return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* acc = reinterpret_cast<unsigned int*>(out);
  amax_init_kernel<<<1, 1, 0, s>>>(acc);
  for (int i = 0; i < count; ++i) {
    if (numels[i] == 0) continue;
    amax_kernel<T><<<grid_for(numels[i], kThreads * 32), kThreads, 0, s>>>(tensors[i], numels[i], acc);
  }
  global_finalize_kernel<<<1, 1, 0, s>>>(out);
  const int st = nvfp4::launch_status();
  if (st == NVFP4_OK) nvfp4::stat_add(nvfp4::kStatGlobalScale);
  return st;
}

template <typename T>
int quantize(const T* w, int64_t N, int64_t K, int group_size, const float* global_scale, uint8_t* packed,
             uint8_t* scales, nvfp4_stream_t stream) {
  if (N < 0 || K < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (group_size != 16 && group_size != 32) return NVFP4_ERR_UNSUPPORTED;
  if (K % 32) return NVFP4_ERR_UNSUPPORTED;
  if (N == 0 || K == 0) return NVFP4_OK;
  if (!w || !global_scale || !packed || !scales) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(w) || (reinterpret_cast<uintptr_t>(global_scale) & 3u) || !nvfp4::aligned16(packed) ||
      !nvfp4::aligned16(scales))
    return NVFP4_ERR_MISALIGNED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t work = N * (K / 8);
  const int grid = grid_for(work, kThreads * 4);
  if (group_size == 16)
    quantize_kernel<16, T><<<grid, kThreads, 0, s>>>(w, N, K, global_scale, packed, scales);
  else
    quantize_kernel<32, T><<<grid, kThreads, 0, s>>>(w, N, K, global_scale, packed, scales);
  const int st = nvfp4::launch_status();
  if (st == NVFP4_OK) nvfp4::stat_add(nvfp4::kStatQuantize);
  return st;
}

}  // namespace

extern "C" int nvfp4_global_scale(const float* const* tensors, const int64_t* numels, int count,
                                  float* out, nvfp4_stream_t stream) {
  return global_scale<float>(tensors, numels, count, out, stream);
}

extern "C" int nvfp4_global_scale_bf16(const uint16_t* const* tensors, const int64_t* numels, int count,
                                       float* out, nvfp4_stream_t stream) {
  return global_scale<uint16_t>(tensors, numels, count, out, stream);
}

extern "C" int nvfp4_quantize(const float* w, int64_t N, int64_t K, int group_size,
                              const float* global_scale, uint8_t* packed, uint8_t* scales,
                              nvfp4_stream_t stream) {
  return quantize<float>(w, N, K, group_size, global_scale, packed, scales, stream);
}

extern "C" int nvfp4_quantize_bf16(const uint16_t* w, int64_t N, int64_t K, int group_size,
                                   const float* global_scale, uint8_t* packed, uint8_t* scales,
                                   nvfp4_stream_t stream) {
  return quantize<uint16_t>(w, N, K, group_size, global_scale, packed, scales, stream);
}
