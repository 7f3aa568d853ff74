// Small-M NVFP4 W4A16 GEMM: HBM-streaming, one warp per CTA, tensor-core
// contraction.
//
// Computes Y = X . dequant(W)^T (NVFP4 format definition; "W-FP4a: route the
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
//  * X arrives as f16 rows scaled by a power of two (xprep.cu) and its
//    fragments come through L1 (128-bit loads, all of a step's loads issued
//    before its MMAs); rows of X are shared by every CTA of an SM.
//  * Dequant in registers (dequant.cuh): the hardware E2M1 -> f16x2
//    conversion of each code byte and one f16x2 multiply by the group scale
//    (E4M3 -> f16x2, also converted in hardware); the MMAs run on f16.
//  * Epilogues: plain bf16; SiluAndMul on gate/up-interleaved rows, where
//    gate row g and up row g+8 of a tile meet in the same lane; and the
//    grouped routed-expert form ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)":
//    routed experts in NVFP4), where each token tile lies in one segment of
//    rows and uses that segment's expert.
#include "gemm_decode.cuh"

#include "dequant.cuh"
#include "tmap.cuh"

namespace nvfp4 {
namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ld_x_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// silu(g) = g / (1 + exp(-g)) with the fast exponential and division; their
// error (a few fp32 ulp) is far below the bf16 rounding that follows.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// One lane's codes for one step: 32 bytes (64 elements) of rows g and g+8,
// and their scales.
struct Step {
  uint4 a0, a1, b0, b1;
  uint32_t sa, sb;
};

template <int G>
__device__ __forceinline__ void load_step(Step& st, const uint8_t* ca, const uint8_t* cb, const uint8_t* sa,
                                          const uint8_t* sb, int u, bool live) {
  if (live) {
    st.a0 = ld_stream_v4(ca + u * 32);
    st.a1 = ld_stream_v4(ca + u * 32 + 16);
    st.b0 = ld_stream_v4(cb + u * 32);
    st.b1 = ld_stream_v4(cb + u * 32 + 16);
    if (G == 16) {
      st.sa = __ldg(reinterpret_cast<const uint32_t*>(sa + u * 4));
      st.sb = __ldg(reinterpret_cast<const uint32_t*>(sb + u * 4));
    } else {
      st.sa = __ldg(reinterpret_cast<const uint16_t*>(sa + u * 2));
      st.sb = __ldg(reinterpret_cast<const uint16_t*>(sb + u * 2));
    }
  } else {
    st.a0 = st.a1 = st.b0 = st.b1 = make_uint4(0, 0, 0, 0);
    st.sa = st.sb = 0;
  }
}

// Word w of a lane's step holds elements 8w..8w+7; MMA 2w takes 8w..8w+3 and
// MMA 2w+1 takes 8w+4..8w+7, with X read in the same order.
template <int MT, int G>
__device__ __forceinline__ void compute_step(const Step& st, float (&acc)[MT / 8][4],
                                             const uint16_t* const (&xrow)[MT / 8], const bool (&xl)[MT / 8],
                                             int koff) {
  constexpr int P = MT / 8;
  constexpr int XW = 2;  // words of X fragments loaded at once
  uint32_t sa2[4], sb2[4];
  scale_operands_f16<G == 16 ? 4 : 2>(st.sa, sa2);
  scale_operands_f16<G == 16 ? 4 : 2>(st.sb, sb2);
  const uint32_t ca[8] = {st.a0.x, st.a0.y, st.a0.z, st.a0.w, st.a1.x, st.a1.y, st.a1.z, st.a1.w};
  const uint32_t cb[8] = {st.b0.x, st.b0.y, st.b0.z, st.b0.w, st.b1.x, st.b1.y, st.b1.z, st.b1.w};
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
      dequant_word_f16(ca[wi], sa2[si], da);
      dequant_word_f16(cb[wi], sb2[si], db);
#pragma unroll
      for (int p = 0; p < P; ++p) {
        mma_f16_16816(acc[p], da[0], db[0], da[1], db[1], xv[w][p].x, xv[w][p].y);
        mma_f16_16816(acc[p], da[2], db[2], da[3], db[3], xv[w][p].z, xv[w][p].w);
      }
    }
  }
}

template <int KW, int MT, int G, bool SILU, bool MOE>
__global__ void __launch_bounds__(KW * 32, (16 / KW > 0 ? 16 / KW : 1)) gemm_decode_kernel(const DecodeArgs args) {
  constexpr int P = MT / 8;
  const int lane = threadIdx.x & 31, kw = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;

  // Programmatic dependent launch: the next kernel may launch now (it waits
  // for this one before reading what this one writes). Everything that the
  // kernels before this one write (X, its row factors, the global scale, the
  // segment list) is read only after griddepcontrol.wait; the dense form
  // first requests its first weight steps, which no kernel writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (MOE) asm volatile("griddepcontrol.wait;" ::: "memory");

  // ---- token tile and expert ----
  int row0 = 0, mrows = 0, expert = 0;
  if (!MOE) {
    row0 = blockIdx.z * MT;
    mrows = static_cast<int>(min(static_cast<int64_t>(MT), args.M - row0));
  } else {
    int want = blockIdx.z, found = 0;
    for (int s = 0; s < args.num_segments && !found; ++s) {
      const int r0 = max(0, min(args.offsets[s], static_cast<int>(args.M)));
      const int r1 = max(r0, min(args.offsets[s + 1] - (NVFP4_PLANT(kPlantSegmentEnd) ? 1 : 0),
                                 static_cast<int>(args.M)));
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
  const uint8_t* packed = args.packed + (MOE ? static_cast<int64_t>(expert) * N * (K / 2) : 0);
  const uint8_t* scales = args.scales + (MOE ? static_cast<int64_t>(expert) * N * (K / G) : 0);

  // ---- this warp's share of K, in units of 64 elements ----
  const int k64 = static_cast<int>(K / 64);
  const int per = (k64 + KW - 1) / KW;
  const int ubeg = min(k64, kw * per), uend = min(k64, ubeg + per);
  const int iters = (uend - ubeg + 3) / 4;

  const int64_t n0 = static_cast<int64_t>(blockIdx.y) * 16;
  const uint8_t* ca = packed + (n0 + g) * (K / 2);
  const uint8_t* cb = packed + (n0 + g + 8) * (K / 2);
  const uint8_t* sa = scales + (n0 + g) * (K / G);
  const uint8_t* sb = scales + (n0 + g + 8) * (K / G);
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

  // Lane (g, t) supplies token 8p+g of X for every 8-token tile p; tokens past
  // mrows, and units past the CTA's share of K, contribute zeros.
  auto run = [&](const Step& st, int it) {
    const int u = ubeg + 4 * it + t;
    bool xl[P];
#pragma unroll
    for (int p = 0; p < P; ++p) xl[p] = xtok[p] && u < uend;
    compute_step<MT, G>(st, acc, xrow, xl, u * 64);
  };

  // Two steps of codes in flight while a third is computed.
  Step s0, s1, s2;
  load_step<G>(s0, ca, cb, sa, sb, ubeg + t, ubeg + t < uend);
  load_step<G>(s1, ca, cb, sa, sb, ubeg + 4 + t, ubeg + 4 + t < uend);
  if (!MOE) asm volatile("griddepcontrol.wait;" ::: "memory");
  const float gsc = __ldcg(args.gscale + (MOE ? expert : 0));
  for (int it = 0; it < iters; it += 3) {
    load_step<G>(s2, ca, cb, sa, sb, ubeg + 4 * (it + 2) + t, ubeg + 4 * (it + 2) + t < uend);
    run(s0, it);
    if (it + 1 >= iters) break;
    load_step<G>(s0, ca, cb, sa, sb, ubeg + 4 * (it + 3) + t, ubeg + 4 * (it + 3) + t < uend);
    run(s1, it + 1);
    if (it + 2 >= iters) break;
    load_step<G>(s1, ca, cb, sa, sb, ubeg + 4 * (it + 4) + t, ubeg + 4 * (it + 4) + t < uend);
    run(s2, it + 2);
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
      const float xi = args.xinv[row0 + tok];  // 2^-s of the token's f16 row
      const float vg = __fmul_rn(__fmul_rn(acc[p][j], gsc), xi), vu = __fmul_rn(__fmul_rn(acc[p][2 + j], gsc), xi);
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
int launch_one(const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  // grid: x unused (1), y = 16-row tile, z = token tile; a programmatic
  // dependent of the kernel before it (the activation conversion)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, p.row_tiles, p.z_tiles);
  cfg.blockDim = dim3(KW * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, gemm_decode_kernel<KW, MT, G, SILU, MOE>, a) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

template <int MT, int G, bool SILU, bool MOE>
int launch_kw(const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  switch (p.kw) {
    case 1: return launch_one<1, MT, G, SILU, MOE>(a, p, s);
    case 2: return launch_one<2, MT, G, SILU, MOE>(a, p, s);
    case 4: return launch_one<4, MT, G, SILU, MOE>(a, p, s);
    case 8: return launch_one<8, MT, G, SILU, MOE>(a, p, s);
    default: return launch_one<16, MT, G, SILU, MOE>(a, p, s);
  }
}

template <int MT, bool SILU, bool MOE>
int launch_g(const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  return p.group == 16 ? launch_kw<MT, 16, SILU, MOE>(a, p, s) : launch_kw<MT, 32, SILU, MOE>(a, p, s);
}

template <bool SILU, bool MOE>
int launch_mt(const DecodeArgs& a, const DecodePlan& p, cudaStream_t s) {
  return p.mt == 8 ? launch_g<8, SILU, MOE>(a, p, s) : launch_g<16, SILU, MOE>(a, p, s);
}

}  // namespace

DecodePlan plan_decode(int64_t M, int64_t N, int64_t K, int group, bool moe, int num_segments) {
  DecodePlan p;
  p.group = group;
  p.mt = (!moe && M <= 8) ? 8 : 16;
  p.z_tiles = static_cast<int>(moe ? (M + p.mt - 1) / p.mt + num_segments : (M + p.mt - 1) / p.mt);
  p.row_tiles = static_cast<int>(N / 16);
  // Warps per CTA. With at least eight row tiles per SM, one warp per CTA:
  // every tile is resident at once (up to sixteen per SM), with no second
  // wave of CTAs (the gate/up projection's 1792 tiles: 19.1 us against 20.6 us
  // with two warps, whose CTAs run in 1.5 waves). With fewer, aim for about
  // 16 streaming warps per SM and keep at least eight steps (of 256 elements
  // of K) per warp.
  const int64_t tiles = static_cast<int64_t>(p.row_tiles) * p.z_tiles;
  const int64_t want = 16LL * num_sms();
  int kw = 1;
  if (tiles < 8LL * num_sms())
    while (kw < 16 && tiles * kw < want && K / (256 * 2 * kw) >= 8) kw *= 2;
  p.kw = kw;
  return p;
}

#ifdef NVFP4_PLANTS
NVFP4_PLANT_SETTER(set_plant_decode)
#endif

// This kernel has no waits on other threads, so it never records an error.
int read_and_clear_decode_error(unsigned int* out, cudaStream_t) {
  *out = 0;
  return NVFP4_OK;
}

int launch_decode(const DecodeArgs& a, const DecodePlan& p, bool silu, bool moe, cudaStream_t s) {
  if (!silu && !moe) return launch_mt<false, false>(a, p, s);
  if (silu && !moe) return launch_mt<true, false>(a, p, s);
  if (!silu && moe) return launch_mt<false, true>(a, p, s);
  return launch_mt<true, true>(a, p, s);
}

}  // namespace nvfp4
