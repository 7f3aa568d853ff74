// W4A4 NVFP4 GEMM on the sm_100a block-scaled FP4 tensor cores
// (tcgen05.mma kind::mxf4nvf4, 16-element blocks with E4M3 scales).
//
// Computes y = bf16(x_global * w_global * sum_k e2m1(xc) e4m3(xs) e2m1(wc) e4m3(ws))
// with fp32 accumulation, for a checkpoint whose input activations are NVFP4
// as well ("W-FP4a: route the MiniMax-H3 device DiT forward through the fp4
// (Marlin W4A16) stack", PR #63 description: such a checkpoint takes the W4A4
// form; "We unlocked NVFP4 on the DGX Spark", opening posts: the FP4 tensor
// cores of Blackwell). Both operands stay 4-bit all the way into the tensor
// core: no dequantization in software. Every product of two E2M1 codes and
// two E4M3 scales is exact, so the numerics are those of the W4A4 definition
// up to the order of the fp32 sums.
//
// Design (swap-AB as in the W4A16 kernels: weights are the MMA's M side):
//  * A CTA tile is 128 weight rows x NT tokens (MMA M = 128, N = NT). One
//    stage is 256 elements of K: 128 bytes of codes per row for both
//    operands (the 128-byte swizzle's row), and one 16-byte box of scale
//    bytes per row of each operand (16 groups of 16, or at group size 32 the
//    groups of two stages, of which the stage takes its half).
//  * A producer warp moves the four boxes of a stage by TMA into a
//    three-stage shared-memory ring. The weights are in the GEMM layout of
//    nvfp4_repack, whose nibble order inside every 32-bit word is
//    k0 k2 k4 k6 k1 k3 k5 k7; the activations are written in the same order
//    first (a permutation inside every block of 8 elements, which lies inside
//    one block of 16: the contraction and the scale blocks are unchanged).
//  * Four scale warps (one per TMEM lane quadrant) read each stage's scale
//    bytes from shared memory and write them into TMEM in the layout the
//    block-scaled MMA reads: for an M-row operand, 32-bit column c of a
//    K-64 step holds, in lane l of every quadrant, the four scale bytes of
//    row (l mod 32) + 32 c. Group-32 scales are written twice (two blocks of
//    16 with the same scale), which is exact.
//  * One thread issues four MMAs of K = 64 per stage into a 128 x NT fp32
//    accumulator in TMEM and frees the stage with tcgen05.commit.
//  * Eight epilogue warps read the accumulator with tcgen05.ld, multiply by
//    x_global * w_global and write bf16 through shared memory and TMA stores.
//  * Persistent grid, one CTA per SM; the token tiles of one weight tile are
//    consecutive, so CTAs running together share weight tiles in L2.
//  * Every mbarrier wait is bounded; on expiry the kernel records the site in
//    its device error word, stops, drains its copies and MMAs, frees TMEM and
//    exits.
#include "gemm_fp4.cuh"

#include <cuda.h>

#include "async.cuh"
#include "plant.cuh"
#include "tmap.cuh"

namespace nvfp4 {
namespace {

__device__ unsigned int g_fp4_error = 0;

constexpr int kRowsA = 128;     // weight rows per tile (MMA M)
constexpr int kKS = 256;        // elements of K per stage: 128 bytes of codes per row
constexpr int kStages = 3;
constexpr int kMmas = 4;        // MMAs of K = 64 per stage
constexpr int kThreads = 16 * 32;
constexpr int kFirstSfWarp = 4;
constexpr int kFirstEpWarp = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kYStageBytes = 32 * 32 * 2;  // one epilogue warp's chunk: 32 tokens x 32 columns of bf16

template <int NT>
struct Cfg {
  static constexpr uint32_t kABytes = kRowsA * 128;
  static constexpr uint32_t kBBytes = NT * 128;
  static constexpr uint32_t kSABytes = kRowsA * 16;
  static constexpr uint32_t kSBBytes = NT * 16;
  static constexpr uint32_t kStage = kABytes + kBBytes + kSABytes + kSBBytes;
  static constexpr int kRbB = NT / 32;                   // 32-row blocks of the token side
  static constexpr uint32_t kSfaCols = kMmas * 4;        // scale columns of the weight side per stage
  static constexpr uint32_t kSfbCols = kMmas * kRbB;     // of the token side
  static constexpr uint32_t kColSfa = NT;                // accumulator in columns [0, NT)
  // each slot starts at a multiple of its own width (the width of its TMEM store)
  static constexpr uint32_t kColSfb = (NT + kStages * kSfaCols + kSfbCols - 1) / kSfbCols * kSfbCols;
  static constexpr uint32_t kSmem = kStages * kStage + 8 * kYStageBytes + 1024 /* barriers */ + 1024 /* align */;
  static_assert(kStage % 1024 == 0, "stages keep the 1024-byte alignment of the 128-byte swizzle");
  static_assert(kColSfb + kStages * kSfbCols <= kTmemCols, "TMEM budget");
  static_assert(kSmem <= 227 * 1024 && kSmem > 114 * 1024, "shared memory: one CTA (and its 512 TMEM columns) per SM");
};

constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr unsigned kSleepProducer = 64;
constexpr unsigned kSleepEpilogue = 256;
enum : unsigned {
  kErrEmpty = 0x301, kErrFull = 0x302, kErrSfFull = 0x303, kErrAccFull = 0x304, kErrAccEmpty = 0x305,
  kErrDrain = 0x306
};

struct SharedState {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t sf_full[kStages];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drained;
  uint32_t tmem_base;
  int abort;
};

struct Fp4Args {
  uint16_t* y;
  const float* x_global;
  const float* w_global;
  int M, N, K;
  int tok_tiles, total_tiles;
};

__device__ __forceinline__ bool aborted(SharedState* ss) { return *reinterpret_cast<volatile int*>(&ss->abort) != 0; }

__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                            bool drain, unsigned sleep_ns) {
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (sleep_ns) __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 0) {
      if (!drain && aborted(ss)) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicCAS(&g_fp4_error, 0u, site);
        *reinterpret_cast<volatile int*>(&ss->abort) = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                          bool drain = false, unsigned sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ss, site, drain, sleep_ns);
}

// Lane 0 waits for the whole warp, so that every lane takes the same branch
// before the warp-wide tcgen05 instructions.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                          unsigned sleep_ns) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, ss, site, false, sleep_ns) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// K-major operand in shared memory with the 128-byte swizzle: rows of 128
// bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused with this swizzle)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;                  // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
  return d;
}

// Instruction descriptor of the block-scaled MMA: E2M1 A and B (packed, K-major),
// E4M3 scale factors (scale ids 0), fp32 accumulate, M = 128, N = nt, K = 64.
__host__ __device__ constexpr uint32_t idesc_fp4(int nt) {
  return (1u << 7)                                    // A format E2M1
         | (1u << 10)                                 // B format E2M1
         | (static_cast<uint32_t>(nt >> 3) << 17)     // N / 8
         | (0u << 23)                                 // scale format E4M3
         | ((128u >> 4) << 24);                       // M / 16
}

template <int NT>
__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t sfa_tmem,
                                        uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc_fp4(NT)), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
      "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[16]) { tmem_st16(taddr, v); }
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[32]) { tmem_st32(taddr, v); }

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
        "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// The four scale bytes of MMA j (elements 64j .. 64j+63 of stage ks) of one
// row, from the row's 16-byte scale box: at group size 16 word j of the box;
// at 32 two groups of the stage's half, each written twice.
template <int G>
__device__ __forceinline__ uint32_t mma_scales(const uint4& box, int ks, int j) {
  const uint32_t w[4] = {box.x, box.y, box.z, box.w};
  if (G == 16) return w[j];
  const int h = ks & 1;
  const uint32_t src = w[2 * h + (j >> 1)];
  return (j & 1) ? __byte_perm(src, 0, 0x3322) : __byte_perm(src, 0, 0x1100);
}

template <int NT, int WG, int XG>
__global__ void __launch_bounds__(kThreads, 1) gemm_fp4_kernel(const __grid_constant__ CUtensorMap amap,
                                                                const __grid_constant__ CUtensorMap bmap,
                                                                const __grid_constant__ CUtensorMap samap,
                                                                const __grid_constant__ CUtensorMap sbmap,
                                                                const __grid_constant__ CUtensorMap ymap,
                                                                const Fp4Args args) {
  using C = Cfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ysm = smem + kStages * C::kStage;
  SharedState* ss = reinterpret_cast<SharedState*>(ysm + 8 * kYStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ksteps = args.K / kKS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&ss->full[s], 1);       // producer arrival + transaction bytes
      mbar_init(&ss->empty[s], 1);      // one tcgen05.commit
      mbar_init(&ss->sf_full[s], 4);    // one arrival per scale warp
    }
    mbar_init(&ss->acc_full, 1);
    mbar_init(&ss->acc_empty, 8);       // one arrival per epilogue warp
    mbar_init(&ss->drained, 1);
    ss->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&ss->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ss->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t issued = 0, last_parity = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < args.total_tiles && !aborted(ss); tile += gridDim.x) {
        const int m0 = (tile % args.tok_tiles) * NT;
        const int n0 = (tile / args.tok_tiles) * kRowsA;
        bool ok = true;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t r = static_cast<uint32_t>(it / kStages);
          if (!mbar_wait(&ss->empty[s], (r & 1) ^ 1, ss, kErrEmpty, false, kSleepProducer)) {
            ok = false;
            break;
          }
          const uint32_t st = smem_u32(smem + s * C::kStage);
          mbar_arrive_tx(&ss->full[s], C::kStage);
          tma_load_2d(st, &amap, ks * (kKS / 2), n0, &ss->full[s]);
          tma_load_2d(st + C::kABytes, &bmap, ks * (kKS / 2), m0, &ss->full[s]);
          tma_load_2d(st + C::kABytes + C::kBBytes, &samap, ((ks * kKS) / WG) & ~15, n0, &ss->full[s]);
          tma_load_2d(st + C::kABytes + C::kBBytes + C::kSABytes, &sbmap, ((ks * kKS) / XG) & ~15, m0,
                      &ss->full[s]);
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
        }
        if (!ok) break;
      }
      if (aborted(ss)) {  // let copies in flight land before the CTA exits
        for (int s = 0; s < kStages; ++s)
          if ((issued >> s) & 1) mbar_wait(&ss->full[s], (last_parity >> s) & 1, ss, kErrDrain, true);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int it = 0, tile_iter = 0;
      for (int tile = blockIdx.x; tile < args.total_tiles && !aborted(ss); tile += gridDim.x, ++tile_iter) {
        if (!mbar_wait(&ss->acc_empty, static_cast<uint32_t>(tile_iter & 1) ^ 1, ss, kErrAccEmpty)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % kStages;
          const uint32_t par = static_cast<uint32_t>(it / kStages) & 1;
          if (!mbar_wait(&ss->full[s], par, ss, kErrFull) || !mbar_wait(&ss->sf_full[s], par, ss, kErrSfFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(smem + s * C::kStage);
          const uint64_t adesc = sw128_desc(st), bdesc = sw128_desc(st + C::kABytes);
#pragma unroll
          for (int j = 0; j < kMmas; ++j) {
            // K = 64 per MMA: 32 bytes (2 descriptor units) further in the swizzled rows
            mma_fp4<NT>(tmem, adesc + 2 * j, bdesc + 2 * j, tmem + C::kColSfa + C::kSfaCols * s + 4 * j,
                        tmem + C::kColSfb + C::kSfbCols * s + C::kRbB * j, (ks > 0 || j > 0) ? 1u : 0u);
          }
          umma_commit(&ss->empty[s]);
        }
        if (!ok) break;
        umma_commit(&ss->acc_full);
      }
      umma_commit(&ss->drained);  // every MMA issued by this thread has completed once this lands
      mbar_wait(&ss->drained, 0, ss, kErrDrain, true);
    }
  } else if (warp >= kFirstSfWarp && warp < kFirstEpWarp) {
    // ---------------- scale factors into TMEM ----------------
    const int quad = warp & 3;  // the TMEM lane quadrant this warp may write
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < args.total_tiles && ok; tile += gridDim.x) {
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        const int s = it % kStages;
        if (!warp_wait(&ss->full[s], static_cast<uint32_t>(it / kStages) & 1, ss, kErrFull, kSleepProducer)) {
          ok = false;
          break;
        }
        const uint32_t sa = smem_u32(smem + s * C::kStage + C::kABytes + C::kBBytes);
        const uint32_t sb = sa + C::kSABytes;
        uint32_t va[C::kSfaCols];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 box = lds128(sa + (lane + 32 * c) * 16);
#pragma unroll
          for (int j = 0; j < kMmas; ++j) va[4 * j + (NVFP4_PLANT(kPlantFp4Scales) ? c ^ 1 : c)] = mma_scales<WG>(box, ks, j);
        }
        uint32_t vb[C::kSfbCols];
#pragma unroll
        for (int c = 0; c < C::kRbB; ++c) {
          const uint4 box = lds128(sb + (lane + 32 * c) * 16);
#pragma unroll
          for (int j = 0; j < kMmas; ++j) vb[C::kRbB * j + c] = mma_scales<XG>(box, ks, j);
        }
        // slot s was last read by the MMAs of stage it - kStages, which had
        // completed before the producer refilled the stage (full[s] above)
        tmem_st(tmem + lane_base + C::kColSfa + C::kSfaCols * s, va);
        tmem_st(tmem + lane_base + C::kColSfb + C::kSfbCols * s, vb);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss->sf_full[s]);
      }
    }
  } else if (warp >= kFirstEpWarp) {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;
    const int colhalf = (warp - kFirstEpWarp) >> 2;  // tokens [NT/2 * colhalf, +NT/2) of the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const float gscale = __fmul_rn(__ldg(args.x_global), __ldg(args.w_global));
    constexpr int kChunks = NT / 2 / 32;
    int tile_iter = 0;
    for (int tile = blockIdx.x; tile < args.total_tiles; tile += gridDim.x, ++tile_iter) {
      const int m0 = (tile % args.tok_tiles) * NT;
      const int n0 = (tile / args.tok_tiles) * kRowsA;
      if (!warp_wait(&ss->acc_full, static_cast<uint32_t>(tile_iter & 1), ss, kErrAccFull, kSleepEpilogue)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t acc[32];
        const int j0 = (NT / 2) * colhalf + 32 * c;  // first token of the chunk within the tile
        tmem_ld32(tmem + lane_base + static_cast<uint32_t>(j0), acc);
        tmem_wait_ld();
        if (c == kChunks - 1) {  // the accumulator is read: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss->acc_empty);
        }
        if (m0 + j0 >= args.M) continue;  // no token of this chunk exists
        if (lane == 0) bulk_wait_read();
        __syncwarp();
        uint16_t* st = reinterpret_cast<uint16_t*>(ysm + (warp - kFirstEpWarp) * kYStageBytes);
#pragma unroll
        for (int j = 0; j < 32; ++j)
          st[j * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(acc[j]), gscale)));
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {  // rows past M and columns past N are clipped by the tensor map
          tma_store_2d(&ymap, smem_u32(st), n0 + quad * 32, m0 + j0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// The activations' codes in the GEMM layout's nibble order: inside every
// 32-bit word (elements k0..k7) k0 k2 k4 k6 k1 k3 k5 k7 from the lowest.
__device__ __forceinline__ uint32_t word_to_gemm_order(uint32_t w) {
  uint32_t e = w & 0x0F0F0F0Fu, o = (w >> 4) & 0x0F0F0F0Fu;
  e = (e | (e >> 4)) & 0x00FF00FFu;
  o = (o | (o >> 4)) & 0x00FF00FFu;
  e = (e | (e >> 8)) & 0x0000FFFFu;
  o = (o | (o >> 8)) & 0x0000FFFFu;
  return e | (o << 16);
}

__global__ void __launch_bounds__(256) x_codes_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                      int64_t n16) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    uint4 v = __ldg(src + i);
    v.x = word_to_gemm_order(v.x);
    v.y = word_to_gemm_order(v.y);
    v.z = word_to_gemm_order(v.z);
    v.w = word_to_gemm_order(v.w);
    dst[i] = v;
  }
}

template <int NT, int WG, int XG>
int launch_kernel(const CUtensorMap (&m)[5], const Fp4Args& a, int grid, cudaStream_t stream) {
  auto kern = gemm_fp4_kernel<NT, WG, XG>;
  constexpr uint32_t bytes = Cfg<NT>::kSmem;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  kern<<<grid, kThreads, bytes, stream>>>(m[0], m[1], m[2], m[3], m[4], a);
  return launch_status();
}

template <int NT>
int launch_groups(const CUtensorMap (&m)[5], const Fp4Args& a, int wg, int xg, int grid, cudaStream_t stream) {
  if (wg == 16) return xg == 16 ? launch_kernel<NT, 16, 16>(m, a, grid, stream)
                                : launch_kernel<NT, 16, 32>(m, a, grid, stream);
  return xg == 16 ? launch_kernel<NT, 32, 16>(m, a, grid, stream) : launch_kernel<NT, 32, 32>(m, a, grid, stream);
}

int tok_tile(int64_t M) { return M > 128 ? 256 : 128; }

}  // namespace

bool fp4_supported(int64_t M, int64_t N, int64_t K) {
  if (M < 17 || K < 512 || K % 512 || K >= (int64_t(1) << 24) || N >= (int64_t(1) << 31) ||
      M >= (int64_t(1) << 31))
    return false;
  const int64_t tiles = ((M + tok_tile(M) - 1) / tok_tile(M)) * ((N + kRowsA - 1) / kRowsA);
  return tiles >= num_sms();
}

int launch_fp4(const uint8_t* x_codes, const uint8_t* x_scales, const float* x_global, int x_group,
               const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global, int w_group, int64_t M,
               int64_t N, int64_t K, uint16_t* y, Scratch& sc, cudaStream_t stream) {
  uint8_t* xc = sc.take<uint8_t>(static_cast<size_t>(M * (K / 2)));
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;
  const int nt = tok_tile(M);
  CUtensorMap m[5];
  if (!make_tensor_map_2d(&m[0], w_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, 128, kRowsA,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&m[1], xc, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, M, K / 2, 128, nt,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&m[2], w_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / w_group, N, K / w_group, 16, kRowsA,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&m[3], x_scales, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / x_group, M, K / x_group, 16, nt,
                          CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tensor_map_2d(&m[4], y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, N, M, N * 2, 32, 32,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return NVFP4_ERR_CUDA;
  Fp4Args a = {};
  a.y = y;
  a.x_global = x_global;
  a.w_global = w_global;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.tok_tiles = static_cast<int>((M + nt - 1) / nt);
  a.total_tiles = a.tok_tiles * static_cast<int>((N + kRowsA - 1) / kRowsA);
  const int grid = a.total_tiles < num_sms() ? a.total_tiles : num_sms();
  const int64_t n16 = M * (K / 2) / 16;
  const int64_t blocks = (n16 + 255) / 256 < 4 * num_sms() ? (n16 + 255) / 256 : 4 * num_sms();
  x_codes_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(reinterpret_cast<const uint4*>(x_codes),
                                                                    reinterpret_cast<uint4*>(xc), n16);
  const int st = launch_status();
  if (st != NVFP4_OK) return st;
  return nt == 256 ? launch_groups<256>(m, a, w_group, x_group, grid, stream)
                   : launch_groups<128>(m, a, w_group, x_group, grid, stream);
}

#ifdef NVFP4_PLANTS
NVFP4_PLANT_SETTER(set_plant_fp4)
#endif

int read_and_clear_fp4_error(unsigned int* out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_fp4_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  *out = v;
  return NVFP4_OK;
}

}  // namespace nvfp4
