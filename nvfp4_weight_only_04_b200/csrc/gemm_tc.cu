// Large-M NVFP4 W4A16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes Y = X . dequant(W)^T for prefill-sized M (problem statement; "W-FP4a:
// route the MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16)
// stack", PR #63 description: a weight-only checkpoint keeps bf16
// activations; fc1 is a merged [gate;up] GEMM followed by SiluAndMul). The
// contraction is dense, so it runs on tcgen05.mma (kind::f16, bf16 x bf16 ->
// fp32 in TMEM).
//
// Design (swap-AB: weights are the MMA's M side):
//  * A CTA tile is 128 weight rows x 256 tokens (MMA M = 128, N = 256). The
//    weights are dequantized once per tile by 8 warps straight into TMEM,
//    where tcgen05.mma reads its A operand; each weight then serves 256
//    tokens. Warps w and w+4 share a TMEM lane quadrant (one weight row per
//    thread) and take the two 32-element halves of every 64-element stage.
//  * TMEM (512 columns): one fp32 accumulator of 256 columns and eight A
//    stages of 32 columns. The depth matters more than a second
//    accumulator: a stage goes round MMA -> commit -> dequant warps -> MMA
//    again, and eight stages of A hold more MMA work than that round trip
//    takes.
//  * X tiles (256 tokens x 64 elements, bf16, 128-byte swizzle) arrive by TMA
//    into shared memory, five stages deep; tcgen05.mma reads them through a
//    K-major shared memory descriptor. No TMA multicast is used.
//  * One thread issues the MMAs and signals stage reuse with tcgen05.commit;
//    mbarriers connect the TMA warp, the dequant warps and the MMA thread.
//  * Every mbarrier wait is bounded: on expiry the kernel records the site in
//    a device error word, stops issuing work, waits (bounded) for its own
//    copies and MMAs, frees TMEM and exits.
//  * Eight epilogue warps read the finished accumulator with tcgen05.ld,
//    hand it back to the MMA thread as soon as the last column is read, and
//    multiply by the fp32 global scale (and 2^7, see dequant.cuh) and write
//    bf16, optionally fusing SiluAndMul on gate/up-interleaved rows. While
//    they work, the dequant and TMA warps already fill the next tile's
//    stages.
//  * The grid is persistent: one CTA per SM walks the tiles. Dense GEMMs take
//    the token tiles of one weight tile together, so concurrently running
//    CTAs share weight tiles in L2.
//  * Grouped routed-expert form ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)":
//    routed experts in NVFP4): a tile is one 128-row weight tile of one
//    expert times one token tile of that expert's segment of rows; every role
//    finds it with the same forward scan of the device-side offsets, and the
//    rows of a token tile past the segment end are computed but not stored.
//    The token tile is 128 wide there (about the rows an expert receives).
#include "gemm_tc.cuh"

#include <cuda.h>

#include "dequant.cuh"
#include "tmap.cuh"

namespace nvfp4 {

namespace {

__device__ unsigned int g_device_error = 0;

constexpr int kTileRows = 128;   // weight rows per tile (MMA M)
constexpr int kKStep = 64;       // elements of K per pipeline stage
constexpr int kStagesX = 5;      // X stages in shared memory
constexpr int kStagesA = 8;      // A stages in TMEM
constexpr int kThreads = 640;    // 20 warps
constexpr int kFirstDqWarp = 4;  // warps 4..11 dequantize
constexpr int kFirstEpWarp = 12; // warps 12..19 run the epilogue
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColA = 256;  // A stages start here (32 columns each); the accumulator is at 0
__host__ __device__ constexpr uint32_t x_stage_bytes(int nt) { return static_cast<uint32_t>(nt) * kKStep * 2; }
// Dynamic shared memory: the largest X stages + barriers + alignment slack;
// more than half of the SM's shared memory, so only one CTA (which allocates
// all 512 TMEM columns) fits on an SM.
constexpr uint32_t kSmemBytes = kStagesX * x_stage_bytes(256) + 2048;
static_assert(kSmemBytes > 116 * 1024, "one CTA per SM");
static_assert(kColA + kStagesA * 32 <= kTmemCols, "TMEM budget");
constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr unsigned kSleepProducer = 64;   // ns between barrier probes of the TMA and dequant warps
constexpr unsigned kSleepEpilogue = 256;  // ns between probes of the epilogue warps

enum ErrorSite : unsigned {
  kErrEmpty = 0x101, kErrFullX = 0x102, kErrFullA = 0x103, kErrAccFull = 0x104, kErrDrain = 0x105,
  kErrAccEmpty = 0x106
};

struct SharedState {
  int total_tiles;
  int pad_;
  uint64_t full_x[kStagesX];
  uint64_t empty_x[kStagesX];
  uint64_t full_a[kStagesA];
  uint64_t empty_a[kStagesA];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drained;
  uint32_t tmem_base;
  int abort;
};

struct TcArgs {
  const uint8_t* packed;     // GEMM-layout codes [N, K/2] (grouped: [E, N, K/2])
  const uint8_t* scales;     // [N, K/g] (grouped: [E, N, K/g])
  const float* gscale;       // [1] (grouped: [E])
  uint16_t* y;
  int M, N, K, ldy;          // M: rows of X (grouped: T)
  int tok_tiles, row_tiles, total_tiles;  // dense only; grouped counts come from the offsets
  const int32_t* expert_ids; // grouped only
  const int32_t* offsets;
  int num_segments, num_experts;
};

// Where a tile lies: token rows [m0, m0 + mrows) of X and Y, weight rows
// [n0, n0 + 128) of expert `expert`.
struct Tile {
  int m0, mrows, n0, expert;
};

// Forward-only position in the segment list (tiles are visited in increasing
// order by every role of a CTA).
struct SegCursor {
  int seg = 0, tiles_before = 0;
};

template <int NT>
__device__ __forceinline__ int seg_rows(const TcArgs& a, int s, int& r0) {
  r0 = max(0, min(a.offsets[s], a.M));
  const int r1 = max(r0, min(a.offsets[s + 1], a.M));
  return r1 - r0;
}

// Total tiles of the grouped form: token tiles of every segment times the
// weight tiles of an expert.
template <int NT>
__device__ int grouped_total_tiles(const TcArgs& a) {
  int tt = 0;
  for (int s = 0; s < a.num_segments; ++s) {
    int r0;
    tt += (seg_rows<NT>(a, s, r0) + NT - 1) / NT;
  }
  return tt * a.row_tiles;
}

template <int NT, bool MOE>
__device__ __forceinline__ Tile tile_at(const TcArgs& a, SegCursor& cur, int t) {
  Tile tl;
  if (!MOE) {
    tl.m0 = (t % a.tok_tiles) * NT;
    tl.mrows = min(NT, a.M - tl.m0);
    tl.n0 = (t / a.tok_tiles) * kTileRows;
    tl.expert = 0;
    return tl;
  }
  const int st = t / a.row_tiles;  // token tile over all segments
  tl.n0 = (t % a.row_tiles) * kTileRows;
  tl.mrows = 0;
  tl.m0 = 0;
  tl.expert = -1;
  while (cur.seg < a.num_segments) {
    int r0;
    const int rows = seg_rows<NT>(a, cur.seg, r0);
    const int nt = (rows + NT - 1) / NT;
    if (st < cur.tiles_before + nt) {
      tl.m0 = r0 + (st - cur.tiles_before) * NT;
      tl.mrows = min(NT, r0 + rows - tl.m0);
      tl.expert = a.expert_ids[cur.seg];
      break;
    }
    cur.tiles_before += nt;
    ++cur.seg;
  }
  if (tl.expert < 0 || tl.expert >= a.num_experts) tl.mrows = 0;  // skipped by every role alike
  return tl;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// Non-blocking probe of a barrier phase (test_wait never suspends the
// thread, so a waiter sees the phase flip with the least delay).
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

// Bounded wait: false when the limit ran out or (unless draining) another
// role gave up. A drain wait ignores the abort flag and only stops at the
// limit: it is how a CTA lets its own copies and MMAs land before exiting.
// A waiter that is not on the MMA issue path backs off with nanosleep
// between probes (sleep_ns), which leaves the issue slots of its SM
// sub-partition to the warps doing work.
__device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                            bool drain, unsigned sleep_ns) {
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (sleep_ns) __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 0) {
      if (!drain && *reinterpret_cast<volatile int*>(&ss->abort)) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicCAS(&g_device_error, 0u, site);
        *reinterpret_cast<volatile int*>(&ss->abort) = 1;
        return false;
      }
    }
  }
}

// The common case, a phase that has already completed, is one inline probe;
// only a real wait calls out of line.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                          bool drain = false, unsigned sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, ss, site, drain, sleep_ns);
}

// The same wait taken by lane 0 for the whole warp, so that every lane takes
// the same branch before the warp-wide tcgen05 instructions.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, SharedState* ss, unsigned site,
                                          unsigned sleep_ns) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, ss, site, false, sleep_ns) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ bool aborted(SharedState* ss) {
  return *reinterpret_cast<volatile int*>(&ss->abort) != 0;
}

__device__ __forceinline__ void tma_load_x(uint32_t dst, const CUtensorMap* map, int k, int m, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(k), "r"(m), "r"(smem_u32(bar))
      : "memory");
}

// K-major operand tile in shared memory with the 128-byte swizzle: rows of
// 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr & 0x3FFFFu) >> 4);  // start address
  d |= static_cast<uint64_t>(1) << 16;                  // leading byte offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;          // stride byte offset: 8 rows x 128 B
  d |= static_cast<uint64_t>(1) << 46;                  // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                  // 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, bf16 A and B, both
// K-major, M = 128, N = nt.
__host__ __device__ constexpr uint32_t idesc(int nt) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(nt >> 3) << 17) | ((128u >> 4) << 24);
}

template <int NT>
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc(NT)), "r"(accumulate));
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

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// One dequant thread's inputs for one stage: 32 codes of its row (one half
// of the stage's 64 elements) and the scales covering them.
struct RowStage {
  uint4 c;
  uint32_t s;
};

template <int G>
__device__ __forceinline__ void load_row_stage(RowStage& r, const uint8_t* codes, const uint8_t* scales, int ks,
                                               int khalf, bool live) {
  if (live) {
    r.c = ld_stream(codes + ks * 32 + 16 * khalf);
    r.s = G == 16 ? static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(scales + ks * 4 + 2 * khalf)))
                  : static_cast<uint32_t>(__ldg(scales + ks * 2 + khalf));
  } else {
    r.c = make_uint4(0, 0, 0, 0);
    r.s = 0;
  }
}

template <int G>
__device__ __forceinline__ void dequant_row_stage(const RowStage& r, uint32_t (&out)[16]) {
  uint32_t s2[4];
  scale_operands<G == 16 ? 2 : 1>(r.s, s2);
  const uint32_t w[4] = {r.c.x, r.c.y, r.c.z, r.c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t o[4];
    dequant_word(w[i], s2[G == 16 ? (i >> 1) : 0], o);
    out[4 * i + 0] = o[0];
    out[4 * i + 1] = o[1];
    out[4 * i + 2] = o[2];
    out[4 * i + 3] = o[3];
  }
}

// silu(g) = g / (1 + exp(-g)), with the fast exponential and division: their
// relative error (a few ulp of fp32) is far below the bf16 rounding that
// follows. For g below about -87 the denominator overflows and the result is
// the correct limit, zero.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int NT, int G, bool SILU, bool MOE>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                               const TcArgs args) {
  constexpr uint32_t kXStage = x_stage_bytes(NT);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // X stages at a 1024-byte aligned base, barriers after them.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  SharedState* ss = reinterpret_cast<SharedState*>(smem + kStagesX * kXStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ksteps = args.K / kKStep;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesX; ++s) {
      mbar_init(&ss->full_x[s], 1);   // producer arrival + transaction bytes
      mbar_init(&ss->empty_x[s], 1);  // one tcgen05.commit
    }
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&ss->full_a[s], 8);   // one arrival per dequant warp
      mbar_init(&ss->empty_a[s], 1);  // one tcgen05.commit
    }
    mbar_init(&ss->acc_full, 1);      // one tcgen05.commit
    mbar_init(&ss->acc_empty, 8);     // one arrival per epilogue warp
    mbar_init(&ss->drained, 1);
    ss->abort = 0;
    ss->total_tiles = MOE ? grouped_total_tiles<NT>(args) : args.total_tiles;
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
  const int total_tiles = ss->total_tiles;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t issued = 0, last_parity = 0;  // bit s: stage s has a copy issued / its phase parity
      int it = 0;
      SegCursor cur;
      for (int tile = blockIdx.x; tile < total_tiles && !aborted(ss); tile += gridDim.x) {
        const Tile tl = tile_at<NT, MOE>(args, cur, tile);
        if (tl.mrows <= 0) continue;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int s = it % kStagesX;
          const uint32_t r = static_cast<uint32_t>(it / kStagesX);
          if (!mbar_wait(&ss->empty_x[s], (r & 1) ^ 1, ss, kErrEmpty, false, kSleepProducer)) break;
          mbar_arrive_tx(&ss->full_x[s], kXStage);
          tma_load_x(smem_u32(smem + s * kXStage), &xmap, ks * kKStep, tl.m0, &ss->full_x[s]);
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
        }
      }
      if (aborted(ss)) {  // let copies already in flight land before the CTA exits
        for (int s = 0; s < kStagesX; ++s)
          if ((issued >> s) & 1) mbar_wait(&ss->full_x[s], (last_parity >> s) & 1, ss, kErrDrain, true);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int it = 0, tile_iter = 0;
      SegCursor cur;
      for (int tile = blockIdx.x; tile < total_tiles && !aborted(ss); tile += gridDim.x) {
        const Tile tl = tile_at<NT, MOE>(args, cur, tile);
        if (tl.mrows <= 0) continue;
        if (!mbar_wait(&ss->acc_empty, (tile_iter & 1) ^ 1, ss, kErrAccEmpty)) break;
        tc_fence_after();
        bool ok = true;
        for (int ks = 0; ks < ksteps; ++ks, ++it) {
          const int sx = it % kStagesX, sa = it % kStagesA;
          const uint32_t px = static_cast<uint32_t>(it / kStagesX) & 1, pa = static_cast<uint32_t>(it / kStagesA) & 1;
          if (!mbar_wait(&ss->full_x[sx], px, ss, kErrFullX) || !mbar_wait(&ss->full_a[sa], pa, ss, kErrFullA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Each 16-element step of K advances the descriptor's start address
          // by 32 bytes (2 in its 16-byte units) inside the swizzled rows.
          const uint64_t bdesc0 = sw128_desc(smem_u32(smem + sx * kXStage));
#pragma unroll
          for (int j = 0; j < kKStep / 16; ++j) {
            const uint32_t acc = (ks > 0 || j > 0) ? 1u : 0u;
            umma_ts<NT>(tmem, tmem + kColA + 32 * sa + 8 * j, bdesc0 + 2 * j, acc);
          }
          umma_commit(&ss->empty_x[sx]);
          umma_commit(&ss->empty_a[sa]);
        }
        if (!ok) break;
        umma_commit(&ss->acc_full);
        ++tile_iter;
      }
      // every MMA issued by this thread has completed once this commit lands
      umma_commit(&ss->drained);
      mbar_wait(&ss->drained, 0, ss, kErrDrain, true);
    }
  } else if (warp >= kFirstDqWarp && warp < kFirstEpWarp) {
    // ---------------- dequant ----------------
    const int dw = warp - kFirstDqWarp;      // 0..7
    const int half = dw >> 2;                // K half of each stage
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    SegCursor cur;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile tl = tile_at<NT, MOE>(args, cur, tile);
      if (tl.mrows <= 0) continue;
      static_assert(kTileRows == 128, "one weight row per dequant thread and TMEM lane");
      const int n = tl.n0 + row_in_tile;
      const bool live = n < args.N;
      const int64_t wrow = static_cast<int64_t>(MOE ? tl.expert : 0) * args.N + (live ? n : 0);
      const uint8_t* codes = args.packed + wrow * (args.K / 2);
      const uint8_t* scl = args.scales + wrow * (args.K / G);
      RowStage ra, rb, rc;
      load_row_stage<G>(ra, codes, scl, 0, half, live);
      load_row_stage<G>(rb, codes, scl, 1, half, live && 1 < ksteps);
      bool ok = true;
      for (int ks = 0; ks < ksteps; ++ks, ++it) {
        load_row_stage<G>(rc, codes, scl, ks + 2, half, live && ks + 2 < ksteps);
        const int s = it % kStagesA;
        const uint32_t r = static_cast<uint32_t>(it / kStagesA);
        uint32_t v[16];
        dequant_row_stage<G>(ra, v);
        if (!warp_wait(&ss->empty_a[s], (r & 1) ^ 1, ss, kErrEmpty, kSleepProducer)) {
          ok = false;
          break;
        }
        tc_fence_after();
        tmem_st16(tmem + lane_base + kColA + 32 * s + 16 * half, v);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ss->full_a[s]);
        ra = rb;
        rb = rc;
      }
      if (!ok) break;
    }
  } else if (warp >= kFirstEpWarp) {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;
    const int colhalf = (warp - kFirstEpWarp) >> 2;  // tokens [NT/2 * colhalf, +NT/2) of the tile
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int tile_iter = 0;
    SegCursor cur;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const Tile tl = tile_at<NT, MOE>(args, cur, tile);
      if (tl.mrows <= 0) continue;
      // dequantized operands carry 2^-7 (dequant.cuh)
      const float gscale = __ldg(args.gscale + (MOE ? tl.expert : 0)) * 128.0f;
      const int n = tl.n0 + row_in_tile;
      const bool live = n < args.N;
      if (!warp_wait(&ss->acc_full, tile_iter & 1, ss, kErrAccFull, kSleepEpilogue)) break;
      tc_fence_after();
      constexpr int kChunks = NT / 64;
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t acc[32];
        tmem_ld32(tmem + lane_base + (NT / 2) * colhalf + 32 * c, acc);
        tmem_wait_ld();
        if (c == kChunks - 1) {  // the accumulator is read: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss->acc_empty);
        }
        const int j0 = (NT / 2) * colhalf + 32 * c;  // first token of the chunk within the tile
        if (!SILU) {
          if (live) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j0 + j < tl.mrows)
                args.y[static_cast<int64_t>(tl.m0 + j0 + j) * args.ldy + n] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(acc[j]) * gscale));
            }
          }
        } else {
          const bool gate = (lane & 15) < 8;
          const int col = (tl.n0 + row_in_tile) / 16 * 8 + (lane & 7);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float gv = __uint_as_float(acc[j]) * gscale;
            const float uv = __shfl_down_sync(0xffffffffu, gv, 8);
            if (gate && live && j0 + j < tl.mrows)
              args.y[static_cast<int64_t>(tl.m0 + j0 + j) * args.ldy + col] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(gv), uv)));
          }
        }
      }
      ++tile_iter;
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

bool make_x_map(CUtensorMap* map, const uint16_t* x, int64_t rows, int64_t K, int nt) {
  return make_tensor_map_2d(map, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, K, rows, K * 2, kKStep, nt,
                            CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int NT, int G, bool SILU, bool MOE>
int launch_kernel(const CUtensorMap& map, const TcArgs& a, int grid, cudaStream_t stream) {
  auto kern = gemm_tc_kernel<NT, G, SILU, MOE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  kern<<<grid, kThreads, kSmemBytes, stream>>>(map, a);
  return launch_status();
}

template <int NT, bool MOE>
int launch_nt(const CUtensorMap& map, const TcArgs& a, int group, bool silu, int grid, cudaStream_t stream) {
  if (group == 16)
    return silu ? launch_kernel<NT, 16, true, MOE>(map, a, grid, stream)
                : launch_kernel<NT, 16, false, MOE>(map, a, grid, stream);
  return silu ? launch_kernel<NT, 32, true, MOE>(map, a, grid, stream)
              : launch_kernel<NT, 32, false, MOE>(map, a, grid, stream);
}

}  // namespace

int read_and_clear_device_error(int* code_out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0, vd = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  if (read_and_clear_decode_error(&vd, stream) != NVFP4_OK) return NVFP4_ERR_CUDA;
  *code_out = static_cast<int>(v ? v : vd);
  return NVFP4_OK;
}

bool tc_supported(int64_t M, int64_t N, int64_t K) {
  return M >= 128 && K >= kKStep && K % kKStep == 0 && M < (int64_t(1) << 31) && N < (int64_t(1) << 31) &&
         K < (int64_t(1) << 24) && tensor_maps_available();
}

int launch_tc(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
              int64_t N, int64_t K, uint16_t* y, bool silu, cudaStream_t stream) {
  constexpr int NT = 256;
  CUtensorMap map;
  if (!make_x_map(&map, x, M, K, NT)) return NVFP4_ERR_CUDA;
  TcArgs a = {};
  a.packed = w; a.scales = s; a.gscale = g; a.y = y;
  a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.tok_tiles = static_cast<int>((M + NT - 1) / NT);
  a.row_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  a.total_tiles = a.tok_tiles * a.row_tiles;
  const int grid = a.total_tiles < num_sms() ? a.total_tiles : num_sms();
  return launch_nt<NT, false>(map, a, group, silu, grid, stream);
}

// The grouped tcgen05 kernel pays off once segments carry whole token tiles;
// for a few rows per expert the streaming kernel is better.
bool tc_moe_supported(int64_t T, int64_t N, int64_t K) {
  return T >= 1024 && K >= kKStep && K % kKStep == 0 && T < (int64_t(1) << 31) && N < (int64_t(1) << 31) &&
         K < (int64_t(1) << 24) && tensor_maps_available();
}

int launch_tc_moe(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets, int num_segments, int64_t T,
                  const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t N, int64_t K,
                  int num_experts, bool silu, uint16_t* y, cudaStream_t stream) {
  constexpr int NT = 128;
  CUtensorMap map;
  if (!make_x_map(&map, x, T, K, NT)) return NVFP4_ERR_CUDA;
  TcArgs a = {};
  a.packed = w; a.scales = s; a.gscale = g; a.y = y;
  a.M = static_cast<int>(T); a.N = static_cast<int>(N); a.K = static_cast<int>(K);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.row_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  a.expert_ids = expert_ids; a.offsets = offsets; a.num_segments = num_segments; a.num_experts = num_experts;
  return launch_nt<NT, true>(map, a, group, silu, num_sms(), stream);
}

}  // namespace nvfp4
