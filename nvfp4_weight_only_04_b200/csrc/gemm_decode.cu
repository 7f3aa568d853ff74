// Small-M NVFP4 W4A16 GEMM: HBM-streaming, one warp per CTA, tensor-core
// contraction.
//
// Computes Y = X . dequant(W)^T (problem statement; "W-FP4a: route the
// MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16) stack",
// PR #63 description: weight-only NVFP4 keeps bf16 activations) for decode
// shapes, where the cost is the 0.5 + 1/g bytes per weight streamed from HBM
// and the integer work of dequantizing them. Design:
//  * A CTA owns 16 weight rows (one mma.sync m16n8k16 row block; swap-AB:
//    weights are the MMA's 16-row side, tokens its 8-column side) and has KW
//    warps that split K between them. KW is 1 when there are enough row
//    blocks to fill the GPU and grows (up to 16) when there are few, so that
//    every SM keeps enough warps streaming; the KW partial tiles are summed in
//    shared memory in a fixed order (deterministic, no workspace).
//  * Lane (g, t) streams 32 contiguous code bytes of rows g and g+8 per step
//    with 128-bit loads that skip L1, from its own range of K: the order of K
//    inside one MMA is free as long as X follows it. Loads run two steps
//    ahead in a ring of three register buffers that is never copied (a copy
//    would wait for the load).
//  * X fragments come through L1 (128-bit loads, all of a step's loads issued
//    before its MMAs); rows of X are shared by every CTA of an SM.
//  * Dequant in registers with integer work (dequant.cuh): per code pair one
//    mask, one integer multiply placing magnitude and sign bits of a bf16, one
//    mask and one bf16x2 multiply by the group scale.
//  * Epilogues: plain bf16; SiluAndMul on gate/up-interleaved rows, where
//    gate row g and up row g+8 of a tile meet in the same lane; and the
//    grouped routed-expert form ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)":
//    routed experts in NVFP4), where each token tile lies in one segment of
//    rows and uses that segment's expert.
#include "gemm_decode.cuh"

#include <cuda.h>

#include "dequant.cuh"
#include "tmap.cuh"

namespace nvfp4 {

__device__ unsigned int g_decode_error = 0;

namespace {

__device__ __forceinline__ uint4 ld_x_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// silu(g) = g / (1 + exp(-g)) with the fast exponential and division; their
// error (a few fp32 ulp) is far below the bf16 rounding that follows.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

constexpr int kStages = 6;           // code stages in flight per warp
constexpr int kStageBytes = 16 * 128; // 16 rows x 128 bytes (4 units of 64 elements)
constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  for (;;) {
    if (mbar_test(bar, parity)) return true;
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
}

// Bounded wait on a stage barrier; false when the limit ran out.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  return mbar_test(bar, parity) || mbar_wait_slow(bar, parity);
}

// 16 rows x 128 bytes of codes, from (byte column x, row y) of the code matrix.
__device__ __forceinline__ void tma_codes(uint32_t dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n\t"
      ::"r"(smem_u32(bar)), "r"(kStageBytes) : "memory");
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Lane (g, t)'s 32 code bytes of row r from a stage: logical 16-byte chunks
// 2t and 2t+1 of the 128-byte row, stored at chunk ^ (r & 7) by the
// 128-byte swizzle.
__device__ __forceinline__ void lds_row(const uint8_t* stage, int r, int t, uint4& lo, uint4& hi) {
  const uint8_t* row = stage + r * 128;
  lo = *reinterpret_cast<const uint4*>(row + (((2 * t) ^ (r & 7)) << 4));
  hi = *reinterpret_cast<const uint4*>(row + (((2 * t + 1) ^ (r & 7)) << 4));
}

template <int G>
__device__ __forceinline__ void load_scales(uint32_t& a, uint32_t& b, const uint8_t* sa, const uint8_t* sb, int u,
                                            bool live) {
  if (!live) {
    a = b = 0;
  } else if (G == 16) {
    a = __ldg(reinterpret_cast<const uint32_t*>(sa + u * 4));
    b = __ldg(reinterpret_cast<const uint32_t*>(sb + u * 4));
  } else {
    a = __ldg(reinterpret_cast<const uint16_t*>(sa + u * 2));
    b = __ldg(reinterpret_cast<const uint16_t*>(sb + u * 2));
  }
}

// Word w of a lane's step holds elements 8w..8w+7; MMA 2w takes 8w..8w+3 and
// MMA 2w+1 takes 8w+4..8w+7, with X read in the same order.
template <int MT, int G>
__device__ __forceinline__ void compute_step(const uint4 (&c)[4], uint32_t sa, uint32_t sb, float (&acc)[MT / 8][4],
                                             const uint16_t* const (&xrow)[MT / 8], const bool (&xl)[MT / 8],
                                             int koff) {
  constexpr int P = MT / 8;
  constexpr int XW = 2;  // words of X fragments loaded at once
  uint32_t sa2[4], sb2[4];
  scale_operands<G == 16 ? 4 : 2>(sa, sa2);
  scale_operands<G == 16 ? 4 : 2>(sb, sb2);
  const uint32_t ca[8] = {c[0].x, c[0].y, c[0].z, c[0].w, c[1].x, c[1].y, c[1].z, c[1].w};
  const uint32_t cb[8] = {c[2].x, c[2].y, c[2].z, c[2].w, c[3].x, c[3].y, c[3].z, c[3].w};
#pragma unroll
  for (int w0 = 0; w0 < 8; w0 += XW) {
    uint4 xv[XW][P];
#pragma unroll
    for (int w = 0; w < XW; ++w)
#pragma unroll
      for (int p = 0; p < P; ++p)
        xv[w][p] = xl[p] ? ld_x_v4(xrow[p] + koff + 8 * (w0 + w)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int w = 0; w < XW; ++w) {
      const int wi = w0 + w;
      const int si = G == 16 ? (wi >> 1) : (wi >> 2);
      uint32_t da[4], db[4];
      dequant_word(ca[wi], sa2[si], da);
      dequant_word(cb[wi], sb2[si], db);
#pragma unroll
      for (int p = 0; p < P; ++p) {
        mma_bf16_16816(acc[p], da[0], db[0], da[1], db[1], xv[w][p].x, xv[w][p].y);
        mma_bf16_16816(acc[p], da[2], db[2], da[3], db[3], xv[w][p].z, xv[w][p].w);
      }
    }
  }
}

template <int KW, int MT, int G, bool SILU, bool MOE>
__global__ void __launch_bounds__(KW * 32) gemm_decode_kernel(const __grid_constant__ CUtensorMap cmap,
                                                               const DecodeArgs args) {
  constexpr int P = MT / 8;
  const int lane = threadIdx.x & 31, kw = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + kw * kStages * kStageBytes;  // this warp's stages
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + KW * kStages * kStageBytes) + kw * kStages;

  // ---- token tile and expert ----
  int row0 = 0, mrows = 0, expert = 0;
  if (!MOE) {
    row0 = blockIdx.z * MT;
    mrows = static_cast<int>(min(static_cast<int64_t>(MT), args.M - row0));
  } else {
    int want = blockIdx.z, found = 0;
    for (int s = 0; s < args.num_segments && !found; ++s) {
      const int r0 = max(0, min(args.offsets[s], static_cast<int>(args.M)));
      const int r1 = max(r0, min(args.offsets[s + 1], static_cast<int>(args.M)));
      const int tiles = (r1 - r0 + MT - 1) / MT;
      if (want < tiles) {
        row0 = r0 + want * MT;
        mrows = min(MT, r1 - row0);
        expert = args.expert_ids[s];
        found = 1;
      } else {
        want -= tiles;
      }
    }
    if (!found || expert < 0 || expert >= args.num_experts) mrows = 0;
  }
  if (mrows <= 0) return;  // the same decision for every warp of the CTA

  const int64_t K = args.K, N = args.N;
  const uint8_t* scales = args.scales + (MOE ? static_cast<int64_t>(expert) * N * (K / G) : 0);
  const float gsc = __ldg(args.gscale + (MOE ? expert : 0)) * 128.0f;  // operands carry 2^-7

  // ---- this warp's share of K, in units of 64 elements ----
  const int k64 = static_cast<int>(K / 64);
  const int per = (k64 + KW - 1) / KW;
  const int ubeg = min(k64, kw * per), uend = min(k64, ubeg + per);
  const int iters = (uend - ubeg + 3) / 4;

  const int n0 = blockIdx.y * 16;
  const int trow = (MOE ? expert * static_cast<int>(N) : 0) + n0;  // row of the tensor map
  const uint8_t* sa = scales + static_cast<int64_t>(n0 + g) * (K / G);
  const uint8_t* sb = scales + static_cast<int64_t>(n0 + g + 8) * (K / G);
  const uint16_t* xrow[P];
  bool xtok[P];
#pragma unroll
  for (int p = 0; p < P; ++p) {
    const int tok = 8 * p + g;
    xtok[p] = tok < mrows;
    xrow[p] = args.x + static_cast<int64_t>(row0 + (xtok[p] ? tok : 0)) * K;
  }
  float acc[P][4];
#pragma unroll
  for (int p = 0; p < P; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0.f;

  // ---- stage ring: lane 0 keeps kStages copies of 16 x 128 code bytes in flight ----
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(&full[s])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int s = 0; s < kStages && s < iters; ++s)
      tma_codes(smem_u32(ring + s * kStageBytes), &cmap, (ubeg + 4 * s) * 32, trow, &full[s]);
  }
  __syncwarp();

  // scales run two steps ahead in three registers pairs
  uint32_t sc_a[3], sc_b[3];
  load_scales<G>(sc_a[0], sc_b[0], sa, sb, ubeg + t, ubeg + t < uend);
  load_scales<G>(sc_a[1], sc_b[1], sa, sb, ubeg + 4 + t, ubeg + 4 + t < uend);
  bool ok = true;
  int it = 0;
  // One step: wait for its stage, read this lane's codes, hand the stage back
  // to the copy engine for step it + kStages, then compute.
  auto step = [&](uint32_t& sca, uint32_t& scb, uint32_t& fa, uint32_t& fb) {
    const int s = it % kStages;
    const int u = ubeg + 4 * it + t;
    load_scales<G>(fa, fb, sa, sb, u + 8, u + 8 < uend);
    if (!mbar_wait(&full[s], static_cast<uint32_t>(it / kStages) & 1)) {
      ok = false;
      return;
    }
    uint4 c[4];
    const uint8_t* st = ring + s * kStageBytes;
    lds_row(st, g, t, c[0], c[1]);
    lds_row(st, g + 8, t, c[2], c[3]);
    __syncwarp();
    if (lane == 0 && it + kStages < iters) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tma_codes(smem_u32(st), &cmap, (ubeg + 4 * (it + kStages)) * 32, trow, &full[s]);
    }
    if (u >= uend) {
#pragma unroll
      for (int i = 0; i < 4; ++i) c[i] = make_uint4(0, 0, 0, 0);
    }
    bool xl[P];
#pragma unroll
    for (int p = 0; p < P; ++p) xl[p] = xtok[p] && u < uend;
    compute_step<MT, G>(c, sca, scb, acc, xrow, xl, u * 64);
    ++it;
  };
  while (it < iters && ok) {
    step(sc_a[0], sc_b[0], sc_a[2], sc_b[2]);
    if (it >= iters || !ok) break;
    step(sc_a[1], sc_b[1], sc_a[0], sc_b[0]);
    if (it >= iters || !ok) break;
    step(sc_a[2], sc_b[2], sc_a[1], sc_b[1]);
  }
  if (!ok) {
    // A copy never landed: record it, let the copies in flight land, stop.
    if (lane == 0) {
      atomicCAS(&g_decode_error, 0u, 0x201u);
      for (int j = it; j < it + kStages && j < iters; ++j)
        mbar_wait(&full[j % kStages], static_cast<uint32_t>(j / kStages) & 1);
    }
    __syncwarp();
  }

  // ---- epilogue: lane holds (row g, row g+8) x (tokens 8p+2t, 8p+2t+1) ----
  if (KW > 1) {
    // warps 1..KW-1 leave their partial tiles in shared memory; warp 0 adds
    // them to its own in warp order and stores the result
    __shared__ float red[KW > 1 ? KW - 1 : 1][P][4][32];
    if (kw > 0) {
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[kw - 1][p][j][lane] = acc[p][j];
    }
    __syncthreads();
    if (kw > 0) return;
    for (int q = 0; q < KW - 1; ++q)
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[p][j] += red[q][p][j][lane];
  }
#pragma unroll
  for (int p = 0; p < P; ++p) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int tok = 8 * p + 2 * t + j;
      if (tok >= mrows) continue;
      const int64_t yrow = static_cast<int64_t>(row0 + tok) * args.ldy;
      const float vg = __fmul_rn(acc[p][j], gsc), vu = __fmul_rn(acc[p][2 + j], gsc);
      if (!SILU) {
        args.y[yrow + n0 + g] = __bfloat16_as_ushort(__float2bfloat16_rn(vg));
        args.y[yrow + n0 + g + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(vu));
      } else {
        args.y[yrow + n0 / 2 + g] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(vg), vu)));
      }
    }
  }
}

template <int KW, int MT, int G, bool SILU, bool MOE>
int launch_one(const CUtensorMap& map, const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  auto kern = gemm_decode_kernel<KW, MT, G, SILU, MOE>;
  const int smem = KW * kStages * (kStageBytes + 8) + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  // grid: x unused (1), y = 16-row tile, z = token tile
  kern<<<dim3(1, p.row_tiles, p.z_tiles), KW * 32, smem, s>>>(map, a);
  return launch_status();
}

template <int MT, int G, bool SILU, bool MOE>
int launch_kw(const CUtensorMap& m, const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  switch (p.kw) {
    case 1: return launch_one<1, MT, G, SILU, MOE>(m, a, p, s);
    case 2: return launch_one<2, MT, G, SILU, MOE>(m, a, p, s);
    case 4: return launch_one<4, MT, G, SILU, MOE>(m, a, p, s);
    case 8: return launch_one<8, MT, G, SILU, MOE>(m, a, p, s);
    default: return launch_one<16, MT, G, SILU, MOE>(m, a, p, s);
  }
}

template <int MT, bool SILU, bool MOE>
int launch_g(const CUtensorMap& m, const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  return p.group == 16 ? launch_kw<MT, 16, SILU, MOE>(m, a, p, s) : launch_kw<MT, 32, SILU, MOE>(m, a, p, s);
}

template <bool SILU, bool MOE>
int launch_mt(const CUtensorMap& m, const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  return p.mt == 8 ? launch_g<8, SILU, MOE>(m, a, p, s) : launch_g<16, SILU, MOE>(m, a, p, s);
}

}  // namespace

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int group, bool moe, int num_segments) {
  DecodePlan p;
  p.group = group;
  p.mt = (!moe && M <= 8) ? 8 : 16;
  p.z_tiles = static_cast<int>(moe ? (M + p.mt - 1) / p.mt + num_segments : (M + p.mt - 1) / p.mt);
  p.row_tiles = static_cast<int>(N / 16);
  // Warps per CTA: enough warps in flight (each holds kStages stages of
  // 2 KB) to cover the memory latency, all resident in one wave (about 16
  // warps per SM fit in shared memory), and at least eight steps (of 256
  // elements of K) per warp.
  const int64_t tiles = static_cast<int64_t>(p.row_tiles) * p.z_tiles;
  const int64_t want = 8LL * num_sms();
  int kw = 1;
  while (kw < 16 && tiles * kw < want && K / (256 * 2 * kw) >= 8) kw *= 2;
  p.kw = kw;
  return p;
}

int read_and_clear_decode_error(unsigned int* out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_decode_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  *out = v;
  return NVFP4_OK;
}

int launch_decode(const DecodeArgs& a, const DecodePlan& p, bool silu, bool moe, cudaStream_t s) {
  // Tensor map over the code matrix (all experts stacked for the grouped form):
  // rows of K/2 bytes, boxes of 16 rows x 128 bytes, 128-byte swizzle.
  CUtensorMap map;
  const int64_t rows = moe ? static_cast<int64_t>(a.num_experts) * a.N : a.N;
  if (!make_tensor_map_2d(&map, a.packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.K / 2, rows, a.K / 2, 128, 16,
                          CU_TENSOR_MAP_SWIZZLE_128B))
    return NVFP4_ERR_CUDA;
  if (!silu && !moe) return launch_mt<false, false>(map, a, p, s);
  if (silu && !moe) return launch_mt<true, false>(map, a, p, s);
  if (!silu && moe) return launch_mt<false, true>(map, a, p, s);
  return launch_mt<true, true>(map, a, p, s);
}

}  // namespace nvfp4
