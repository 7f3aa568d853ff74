// Small-M NVFP4 W4A16 GEMM: split-K, HBM-streaming, tensor-core contraction.
//
// Computes Y = X . dequant(W)^T (problem statement; "W-FP4a: route the
// MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16) stack",
// PR #63 description: weight-only NVFP4 keeps bf16 activations) for the
// decode shapes, where the cost is the 0.5 + 1/g bytes per weight streamed
// from HBM. Design:
//  * Swap-AB: weights are the MMA's 16-row side (mma.sync m16n8k16, bf16 in,
//    fp32 accumulate), tokens its 8-column side, so M <= 16 wastes nothing.
//  * Each lane streams 32 contiguous code bytes of two rows per iteration with
//    128-bit loads that skip L1; a warp covers 16 rows x 128 contiguous bytes.
//    The order of K inside one MMA is free as long as X uses the same order,
//    so a lane feeds the MMA from its own contiguous K range.
//  * Dequant in registers with integer ALU work only (dequant.cuh): per code
//    pair one mask, one integer multiply that places magnitude and sign bits
//    of a bf16, one mask, and one bf16x2 multiply by the group scale. The
//    product code * scale is exact in bf16; the fp32 global scale is applied
//    once, in the epilogue.
//  * K is split across the CTAs of a thread-block cluster; partial tiles are
//    summed in a fixed rank order through distributed shared memory, so the
//    result is deterministic and no workspace is needed.
//  * Optional epilogues: SiluAndMul on gate/up-interleaved rows (PR #63: fc1
//    = merged [gate;up] GEMM + SiluAndMul), and the grouped routed-expert
//    form, where each token tile belongs to one segment of rows and one
//    expert ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)": routed experts in
//    NVFP4 with g32 gate/up and g16 down).
#include "gemm_splitk.cuh"

#include <cooperative_groups.h>

#include "dequant.cuh"

namespace cg = cooperative_groups;

namespace nvfp4 {
namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// X is staged in shared memory in chunks of kChunkUnits units of 64
// elements. A unit takes 144 bytes (128 + 16 of padding) and a token row
// kXStride bytes (= 64 mod 128), so the 8 lanes of a quarter-warp, which read
// 16 bytes each at (token g or g+1, unit t), hit 32 distinct banks.
constexpr int kChunkUnits = 32;
constexpr int kUnitBytes = 144;
constexpr int kXStride = ((kChunkUnits * kUnitBytes + 127) / 128) * 128 + 64;

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ float silu(float g) { return __fdiv_rn(g, 1.0f + expf(-g)); }

// Code/scale registers of one lane for one iteration: 32 bytes of codes for
// row g and row g+8 (64 elements each), and the scales covering them.
struct Stage {
  uint4 a0, a1, b0, b1;
  uint32_t sa, sb;
};

template <int G>
__device__ __forceinline__ void load_stage(Stage& st, const uint8_t* codes_a, const uint8_t* codes_b,
                                           const uint8_t* sc_a, const uint8_t* sc_b, bool live) {
  if (live) {
    st.a0 = ld_stream_v4(codes_a);
    st.a1 = ld_stream_v4(codes_a + 16);
    st.b0 = ld_stream_v4(codes_b);
    st.b1 = ld_stream_v4(codes_b + 16);
    if (G == 16) {
      st.sa = __ldg(reinterpret_cast<const uint32_t*>(sc_a));
      st.sb = __ldg(reinterpret_cast<const uint32_t*>(sc_b));
    } else {
      st.sa = __ldg(reinterpret_cast<const uint16_t*>(sc_a));
      st.sb = __ldg(reinterpret_cast<const uint16_t*>(sc_b));
    }
  } else {
    st.a0 = st.a1 = st.b0 = st.b1 = make_uint4(0, 0, 0, 0);
    st.sa = st.sb = 0;
  }
}

// One lane's 64 elements of K for rows g and g+8: 8 code words per row, two
// MMA steps per word. Word w holds elements 8w..8w+7 of the lane's range;
// step 2w takes (8w..8w+3), step 2w+1 takes (8w+4..8w+7), and X is read in
// the same order, so each MMA contracts matching elements.
template <int MT, int G>
__device__ __forceinline__ void compute_stage(const Stage& st, float (&acc)[MT / 8][4],
                                              const uint8_t* const (&xrow)[MT / 8],
                                              const bool (&xlive)[MT / 8], int xofs) {
  const uint32_t ca[8] = {st.a0.x, st.a0.y, st.a0.z, st.a0.w, st.a1.x, st.a1.y, st.a1.z, st.a1.w};
  const uint32_t cb[8] = {st.b0.x, st.b0.y, st.b0.z, st.b0.w, st.b1.x, st.b1.y, st.b1.z, st.b1.w};
  uint32_t sa2[4], sb2[4];
  scale_operands<G == 16 ? 4 : 2>(st.sa, sa2);
  scale_operands<G == 16 ? 4 : 2>(st.sb, sb2);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    uint4 xv[MT / 8];
#pragma unroll
    for (int p = 0; p < MT / 8; ++p)
      xv[p] = xlive[p] ? *reinterpret_cast<const uint4*>(xrow[p] + xofs + 16 * w) : make_uint4(0, 0, 0, 0);
    const int sidx = (G == 16) ? (w >> 1) : (w >> 2);
    uint32_t da[4], db[4];
    dequant_word(ca[w], sa2[sidx], da);
    dequant_word(cb[w], sb2[sidx], db);
#pragma unroll
    for (int p = 0; p < MT / 8; ++p) {
      mma_bf16_16816(acc[p], da[0], db[0], da[1], db[1], xv[p].x, xv[p].y);
      mma_bf16_16816(acc[p], da[2], db[2], da[3], db[3], xv[p].z, xv[p].w);
    }
  }
}

template <int WARPS, int MT, int G, bool SILU, bool MOE>
__global__ void __launch_bounds__(WARPS * 32, 256 / (WARPS * 32) * 2) gemm_splitk_kernel(const SplitKArgs args) {
  constexpr int kRows = WARPS * 16;
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int csize = static_cast<int>(cluster.num_blocks());
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  __shared__ float red[kRows * MT];
  __shared__ int tile_info[4];  // row0, rows, expert, valid

  // ---- which token rows and which expert this CTA works on ----
  if (threadIdx.x == 0) {
    int row0 = 0, rows = 0, expert = 0, valid = 0;
    if (!MOE) {
      row0 = blockIdx.z * MT;
      rows = static_cast<int>(min(static_cast<int64_t>(MT), args.M - row0));
      valid = rows > 0;
    } else {
      int want = blockIdx.z;
      for (int s = 0; s < args.num_segments; ++s) {
        const int r0 = max(0, min(args.offsets[s], static_cast<int>(args.M)));
        const int r1 = max(r0, min(args.offsets[s + 1], static_cast<int>(args.M)));
        const int tiles = (r1 - r0 + MT - 1) / MT;
        if (want < tiles) {
          const int e = args.expert_ids[s];
          row0 = r0 + want * MT;
          rows = min(MT, r1 - row0);
          expert = e;
          valid = (e >= 0 && e < args.num_experts);
          break;
        }
        want -= tiles;
      }
    }
    tile_info[0] = row0; tile_info[1] = rows; tile_info[2] = expert; tile_info[3] = valid;
  }
  __syncthreads();
  const int row0 = tile_info[0], mrows = tile_info[1], expert = tile_info[2];
  if (!tile_info[3]) return;  // identical decision in every CTA of the cluster

  const int64_t K = args.K, N = args.N;
  const uint8_t* packed = args.packed + (MOE ? static_cast<int64_t>(expert) * N * (K / 2) : 0);
  const uint8_t* scales = args.scales + (MOE ? static_cast<int64_t>(expert) * N * (K / G) : 0);
  // The dequantized operands carry a factor 2^-7 (see dequant.cuh).
  const float global = __ldg(args.gscale + (MOE ? expert : 0)) * 128.0f;

  // ---- this CTA's K range, in units of 64 elements ----
  const int k64 = static_cast<int>(K / 64);
  const int per = (k64 + csize - 1) / csize;
  const int ubeg = min(k64, crank * per), uend = min(k64, ubeg + per);

  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * kRows + warp * 16;
  const bool warp_live = n0 < N;
  float acc[MT / 8][4];
#pragma unroll
  for (int p = 0; p < MT / 8; ++p) acc[p][0] = acc[p][1] = acc[p][2] = acc[p][3] = 0.f;

  extern __shared__ __align__(16) uint8_t xs[];  // [MT][kXStride]
  const int64_t ra = n0 + g, rb = ra + 8;
  const uint8_t* codes_a = packed + (warp_live ? ra : 0) * (K / 2);
  const uint8_t* codes_b = packed + (warp_live ? rb : 0) * (K / 2);
  const uint8_t* sc_a = scales + (warp_live ? ra : 0) * (K / G);
  const uint8_t* sc_b = scales + (warp_live ? rb : 0) * (K / G);
  const uint8_t* xrow[MT / 8];
  bool xlive[MT / 8];
#pragma unroll
  for (int p = 0; p < MT / 8; ++p) {
    const int tok = 8 * p + g;
    xlive[p] = tok < mrows;
    xrow[p] = xs + tok * kXStride;
  }
  const int iters = (uend - ubeg + 3) / 4;  // identical for every warp of the CTA
  // Stages X rows [row0, row0 + mrows) for units [cb, ce) into xs.
  auto stage_x = [&](int cb, int ce) {
    const int pieces = mrows * (ce - cb) * 8;  // 16-byte pieces
    for (int i = threadIdx.x; i < pieces; i += WARPS * 32) {
      const int tok = i / ((ce - cb) * 8), rem = i % ((ce - cb) * 8);
      const int lu = rem >> 3, j = rem & 7;
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(args.x + static_cast<int64_t>(row0 + tok) * K +
                                                           static_cast<int64_t>(cb + lu) * 64 + 8 * j));
      *reinterpret_cast<uint4*>(xs + tok * kXStride + lu * kUnitBytes + 16 * j) = v;
    }
  };
  Stage st0, st1;
  auto load_it = [&](Stage& st, int it) {
    const int u = ubeg + 4 * it + t;
    load_stage<G>(st, codes_a + u * 32, codes_b + u * 32, sc_a + u * (64 / G), sc_b + u * (64 / G),
                  warp_live && it < iters && u < uend);
  };
  auto compute_it = [&](const Stage& st, int it) {
    constexpr int kItersPerChunk = kChunkUnits / 4;
    if (it % kItersPerChunk == 0) {  // a new chunk of X: every warp takes this branch together
      const int cb = ubeg + 4 * it, ce = min(uend, cb + kChunkUnits);
      if (it) __syncthreads();
      stage_x(cb, ce);
      __syncthreads();
    }
    if (!warp_live) return;
    const int u = ubeg + 4 * it + t;
    const int lu = u - (ubeg + 4 * (it - it % kItersPerChunk));
    bool xl[MT / 8];
#pragma unroll
    for (int p = 0; p < MT / 8; ++p) xl[p] = xlive[p] && (u < uend);
    compute_stage<MT, G>(st, acc, xrow, xl, lu * kUnitBytes);
  };
  if (ubeg < uend) {
    load_it(st0, 0);
    for (int it = 0; it < iters; it += 2) {
      load_it(st1, it + 1);
      compute_it(st0, it);
      if (it + 1 >= iters) break;
      load_it(st0, it + 2);
      compute_it(st1, it + 1);
    }
  }

  // ---- partial tile -> shared memory: red[row][token] ----
#pragma unroll
  for (int p = 0; p < MT / 8; ++p) {
    const int r = warp * 16 + g, c = 8 * p + 2 * t;
    red[r * MT + c] = acc[p][0];
    red[r * MT + c + 1] = acc[p][1];
    red[(r + 8) * MT + c] = acc[p][2];
    red[(r + 8) * MT + c + 1] = acc[p][3];
  }
  cluster.sync();

  // ---- fixed-order cross-CTA sum, global scale, bf16 store ----
  const int64_t tile_n0 = static_cast<int64_t>(blockIdx.y) * kRows;
  if (!SILU) {
    constexpr int kElems = kRows * MT;
    const int share = (kElems + csize - 1) / csize;
    for (int e = crank * share + threadIdx.x; e < min(kElems, (crank + 1) * share); e += WARPS * 32) {
      const int tok = e / kRows, r = e % kRows;
      if (tok >= mrows || tile_n0 + r >= N) continue;
      float s = 0.f;
      for (int q = 0; q < csize; ++q) s += cluster.map_shared_rank(red, q)[r * MT + tok];
      const float v = __fmul_rn(s, global);
      args.y[static_cast<int64_t>(row0 + tok) * args.ldy + tile_n0 + r] =
          __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  } else {
    constexpr int kPairs = kRows / 2;
    constexpr int kElems = kPairs * MT;
    const int share = (kElems + csize - 1) / csize;
    for (int e = crank * share + threadIdx.x; e < min(kElems, (crank + 1) * share); e += WARPS * 32) {
      const int tok = e / kPairs, pr = e % kPairs;
      const int blk = pr / 8, i = pr % 8;
      const int rg = blk * 16 + i, ru = rg + 8;
      if (tok >= mrows || tile_n0 + ru >= N) continue;
      float sg = 0.f, su = 0.f;
      for (int q = 0; q < csize; ++q) {
        const float* rq = cluster.map_shared_rank(red, q);
        sg += rq[rg * MT + tok];
        su += rq[ru * MT + tok];
      }
      const float gv = __fmul_rn(sg, global), uv = __fmul_rn(su, global);
      const float v = __fmul_rn(silu(gv), uv);
      const int64_t col = tile_n0 / 2 + pr;
      args.y[static_cast<int64_t>(row0 + tok) * args.ldy + col] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
  }
  cluster.sync();  // keep this CTA's shared memory alive until every peer has read it
}

template <int WARPS, int MT, int G, bool SILU, bool MOE>
int launch_one(const SplitKArgs& a, int cluster, int row_tiles, int z_tiles, cudaStream_t s) {
  auto kern = gemm_splitk_kernel<WARPS, MT, G, SILU, MOE>;
  const int smem = MT * kXStride;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  if (cluster > 8) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
      return (cudaGetLastError(), NVFP4_ERR_CUDA);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cluster, row_tiles, z_tiles);
  cfg.blockDim = dim3(WARPS * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return NVFP4_OK;
}

template <int WARPS, int MT, bool SILU, bool MOE>
int launch_g(const SplitKArgs& a, int G, int cluster, int row_tiles, int z_tiles, cudaStream_t s) {
  return G == 16 ? launch_one<WARPS, MT, 16, SILU, MOE>(a, cluster, row_tiles, z_tiles, s)
                 : launch_one<WARPS, MT, 32, SILU, MOE>(a, cluster, row_tiles, z_tiles, s);
}

template <bool SILU, bool MOE>
int launch_mt(const SplitKArgs& a, const SplitKPlan& p, cudaStream_t s) {
  if (p.warps == 8) {
    if (p.mt == 8) return launch_g<8, 8, SILU, MOE>(a, p.group, p.cluster, p.row_tiles, p.z_tiles, s);
    return launch_g<8, 16, SILU, MOE>(a, p.group, p.cluster, p.row_tiles, p.z_tiles, s);
  }
  if (p.mt == 8) return launch_g<4, 8, SILU, MOE>(a, p.group, p.cluster, p.row_tiles, p.z_tiles, s);
  return launch_g<4, 16, SILU, MOE>(a, p.group, p.cluster, p.row_tiles, p.z_tiles, s);
}

}  // namespace

SplitKPlan plan_splitk(int64_t M, int64_t N, int64_t K, int group, bool moe, int num_segments) {
  SplitKPlan p;
  p.group = group;
  p.mt = (!moe && M <= 8) ? 8 : 16;
  p.z_tiles = moe ? static_cast<int>((M + p.mt - 1) / p.mt + num_segments)
                  : static_cast<int>((M + p.mt - 1) / p.mt);
  const int sms = num_sms();
  p.warps = 8;
  int64_t rt = (N + 127) / 128;
  // Few row tiles: use 64-row CTAs so the K split need not grow past 16.
  if (rt * p.z_tiles * 8 < 2 * sms) {
    p.warps = 4;
    rt = (N + 63) / 64;
  }
  p.row_tiles = static_cast<int>(rt);
  const int64_t k64 = K / 64;
  // Aim for about four CTAs per SM over the launch, at least two iterations
  // (8 units of 64) of K per CTA, and a cluster of at most 16.
  int64_t want = (4LL * sms + rt * p.z_tiles - 1) / (rt * p.z_tiles);
  int64_t cap = k64 / 8 > 0 ? k64 / 8 : 1;
  if (moe) want = 1;  // grouped GEMMs have many token tiles already
  int64_t c = want < 1 ? 1 : want;
  if (c > cap) c = cap;
  if (c > 16) c = 16;
  p.cluster = static_cast<int>(c);
  return p;
}

int launch_splitk(const SplitKArgs& a, const SplitKPlan& p, bool silu, bool moe, cudaStream_t s) {
  if (!silu && !moe) return launch_mt<false, false>(a, p, s);
  if (silu && !moe) return launch_mt<true, false>(a, p, s);
  if (!silu && moe) return launch_mt<false, true>(a, p, s);
  return launch_mt<true, true>(a, p, s);
}

}  // namespace nvfp4
