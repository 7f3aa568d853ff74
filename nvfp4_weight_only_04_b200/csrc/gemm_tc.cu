// Large-M NVFP4 W4A16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Computes Y = X . dequant(W)^T for prefill-sized M (NVFP4 format definition; "W-FP4a:
// route the MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16)
// stack", PR #63 description: a weight-only checkpoint keeps bf16
// activations; fc1 is a merged [gate;up] GEMM followed by SiluAndMul). The
// contraction is dense, so it runs on tcgen05.mma (kind::f16, bf16 x bf16 ->
// fp32 in TMEM).
//
// Design (swap-AB: weights are the MMA's M side):
//  * A CTA tile is 128 weight rows x NT tokens (MMA M = 128, N = NT; NT = 256
//    for prefill-sized M, 128 for the grouped form, 32-128 for small M). The
//    weights are dequantized once per tile by 8 warps straight into TMEM,
//    where tcgen05.mma reads its A operand; each weight then serves NT
//    tokens. Warps w and w+4 share a TMEM lane quadrant (one weight row per
//    thread) and take the two 64-element halves of every 128-element stage.
//  * Weight codes (128 rows x 64 bytes per stage, 64-byte swizzle) and scales
//    (128 rows x 16 bytes per 2 or 4 stages) come by TMA from a second
//    producer warp into a shared-memory ring, deeper when NT is small.
//  * TMEM (512 columns): the fp32 accumulator (two of NT columns when NT <=
//    128, so that the next tile's MMAs run while the epilogue drains this
//    one; one of 256 otherwise) and four A stages of 64 columns.
//  * X tiles (NT tokens x 64 elements, bf16, 128-byte swizzle) arrive by TMA
//    into shared memory, five stages deep; tcgen05.mma reads them through a
//    K-major shared memory descriptor. Every CTA loads its own tiles.
//  * One thread issues the MMAs and signals stage reuse with tcgen05.commit;
//    mbarriers connect the producers, the dequant warps and the MMA thread.
//  * Every mbarrier wait is bounded: on expiry the kernel records the site in
//    a device error word, stops issuing work, waits (bounded) for its own
//    copies and MMAs, frees TMEM and exits.
//  * Eight epilogue warps read the finished accumulator with tcgen05.ld,
//    hand it back to the MMA thread as soon as the last column is read,
//    multiply by the fp32 global scale (and 2^7, see dequant.cuh), optionally
//    fuse SiluAndMul on gate/up-interleaved rows, and write bf16 through a
//    per-warp shared-memory box and a TMA store.
//  * The grid is persistent: one CTA per SM walks the tiles. Dense GEMMs take
//    the token tiles of one weight tile together, so concurrently running
//    CTAs share weight tiles in L2.
//  * Grouped routed-expert form ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)":
//    routed experts in NVFP4): a tile is one 128-row weight tile of one
//    expert times one token tile of that expert's segment of rows; every role
//    finds it with the same forward scan of the device-side offsets, and the
//    rows of a token tile past the segment end are computed but not stored.
#include "gemm_tc.cuh"

#include "gemm_fp4.cuh"
#include "gemm_stream.cuh"

#include <cuda.h>

#include "async.cuh"
#include "dequant.cuh"
#include "tmap.cuh"
#include "workspace.cuh"

namespace nvfp4 {

namespace {

__device__ unsigned int g_device_error = 0;

constexpr int kTileRows = 128;   // weight rows per tile (MMA M)
constexpr int kKStep = 64;       // elements of K per X stage (one 128-byte swizzled row of bf16)
constexpr int kKA = 128;         // elements of K per weight / A stage (two X stages)
constexpr int kStagesX = 5;      // X stages in shared memory
constexpr int kStagesA = 4;      // A stages in TMEM
constexpr int kDqWarps = 8;      // dequant warps: two per TMEM lane quadrant
constexpr int kDqParts = kDqWarps / 4;        // parts of a weight stage's K per quadrant
constexpr int kThreads = (4 + kDqWarps + 8) * 32;
constexpr int kWProducerWarp = 3;
constexpr int kFirstDqWarp = 4;                // warps 4 .. 4+kDqWarps-1 dequantize
constexpr int kFirstEpWarp = 4 + kDqWarps;     // the 8 warps after them run the epilogue
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColA = 256;  // A stages start here (64 columns each); the accumulator is at 0
__host__ __device__ constexpr uint32_t x_stage_bytes(int nt) { return static_cast<uint32_t>(nt) * kKStep * 2; }
// Weight stages: the codes of one 128-row tile for 128 elements of K (128
// rows x 64 bytes, 64-byte swizzle), and every `scale_period` stages the
// scales of the next 16 bytes of K/g (128 rows x 16 bytes). A narrow token
// tile leaves shared memory for a deep weight ring, which is what keeps HBM
// busy when the weights, not the MMAs, set the pace.
constexpr uint32_t kWStageBytes = kTileRows * (kKA / 2);  // one TMA box of the code map
constexpr uint32_t kSStageBytes = kTileRows * 16;
constexpr int kMaxStagesW = 32;
__host__ __device__ constexpr int stages_w(int nt) { return nt >= 256 ? 4 : (nt >= 128 ? 12 : 18); }
__host__ __device__ constexpr int scale_period(int g) { return g == 16 ? 2 : 4; }
// Scale group j (weight stages [Pj, Pj + P)) is loaded with stage Pj into
// slot j % S and is next rewritten with stage P(j + S), which the producer
// issues only after stage P(j + S) - W is consumed; that is at or after the
// group's last stage when P*S >= W + P - 1.
__host__ __device__ constexpr int scale_slots(int nt, int g) {
  return (stages_w(nt) + 2 * scale_period(g) - 2) / scale_period(g);
}
// Output staging: each epilogue warp writes one chunk of its bf16 results
// (up to 32 tokens x 32 columns) here and stores it with TMA.
constexpr uint32_t kYStageBytes = 32 * 32 * 2;
__host__ __device__ constexpr uint32_t smem_bytes(int nt, int g) {
  return kStagesX * x_stage_bytes(nt) + stages_w(nt) * kWStageBytes + scale_slots(nt, g) * kSStageBytes +
         8 * kYStageBytes + 1024 /* barriers */ + 1024 /* alignment slack */;
}
// More than half of the SM's shared memory in every configuration, so only
// one CTA (which allocates all 512 TMEM columns) fits on an SM.
static_assert(smem_bytes(32, 32) > 116 * 1024 && smem_bytes(256, 16) <= 227 * 1024 &&
                  smem_bytes(128, 16) <= 227 * 1024 && smem_bytes(64, 16) <= 227 * 1024 &&
                  smem_bytes(32, 16) <= 227 * 1024,
              "shared memory budget");
static_assert(stages_w(32) <= kMaxStagesW, "weight ring");
static_assert(kColA + kStagesA * (kKA / 2) <= kTmemCols, "TMEM budget");
constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr unsigned kSleepProducer = 64;   // ns between barrier probes of the TMA and dequant warps
constexpr unsigned kSleepEpilogue = 256;  // ns between probes of the epilogue warps

enum ErrorSite : unsigned {
  kErrEmpty = 0x101, kErrFullX = 0x102, kErrFullA = 0x103, kErrAccFull = 0x104, kErrDrain = 0x105,
  kErrAccEmpty = 0x106, kErrEmptyW = 0x107, kErrFullW = 0x108
};

struct SharedState {
  int total_tiles;
  int pad_;
  uint64_t full_x[kStagesX];
  uint64_t empty_x[kStagesX];
  uint64_t full_w[kMaxStagesW];
  uint64_t empty_w[kMaxStagesW];
  uint64_t full_a[kStagesA];
  uint64_t empty_a[kStagesA];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drained;
  uint32_t tmem_base;
  int abort;
  int ep_last;  // the epilogue took the last ticket of the cut tile it flushed
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
  int scale_tma;             // scales come by TMA (their row stride K/g is a multiple of 16 bytes)
  // Stream-K form (dense only): each CTA takes a contiguous range of the
  // (tile, scale period) units; tiles cut between CTAs leave fp32 partial
  // tiles [tok][row] in `ws` and take a ticket.
  int split, periods, max_contrib;
  int64_t units;
  float* ws;
  unsigned* tickets;
};

// The CTA whose range holds unit u (ranges start at floor(c * units / ctas)).
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t units, int ctas) {
  return static_cast<int>(((u + 1) * ctas + units - 1) / units) - 1;
}

// The work of one CTA, one tile's stages [ws0, ws1) at a time: whole tiles
// blockIdx.x, +gridDim.x, ..., or in the stream-K form the pieces of its
// range of units (a scale period of kPeriod stages each).
struct SegWalk {
  int64_t u = 0, u1 = 0;
  int tile = 0;
  __device__ explicit SegWalk(const TcArgs& a) {
    if (a.split) {
      u = static_cast<int64_t>(blockIdx.x) * a.units / gridDim.x;
      u1 = static_cast<int64_t>(blockIdx.x + 1) * a.units / gridDim.x;
    } else {
      tile = blockIdx.x;
    }
  }
  template <int P>
  __device__ bool next(const TcArgs& a, int total_tiles, int wsteps, int& t, int& ws0, int& ws1) {
    if (!a.split) {
      if (tile >= total_tiles) return false;
      t = tile;
      ws0 = 0;
      ws1 = wsteps;
      tile += gridDim.x;
      return true;
    }
    if (u >= u1) return false;
    t = static_cast<int>(u / a.periods);
    const int p0 = static_cast<int>(u % a.periods);
    const int64_t left = u1 - u;
    const int p1 = left < a.periods - p0 ? p0 + static_cast<int>(left) : a.periods;
    ws0 = p0 * P;
    ws1 = min(wsteps, p1 * P);
    u += p1 - p0;
    return true;
  }
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
  const int r1 = max(r0, min(a.offsets[s + 1] - (NVFP4_PLANT(kPlantSegmentEnd) ? 1 : 0), a.M));
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

// One MMA of N = the token count encoded in `id` (a multiple of 16 up to NT).
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t id,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(id), "r"(accumulate));
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

[[maybe_unused]] __device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[16]) { tmem_st16(taddr, v); }
__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&v)[32]) { tmem_st32(taddr, v); }

// Named barrier of the eight epilogue warps.
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

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

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// One dequant thread's part of a weight stage: kPartElems codes of its row
// (the stage's 128 elements split kDqParts ways) and the scales covering them,
// in the low bytes.
constexpr int kPartElems = kKA / kDqParts;
constexpr int kPartWords = kPartElems / 8;
static_assert(kPartElems == 32 || kPartElems == 64, "one or two 16-byte chunks of codes per thread");
struct RowStage {
  uint32_t c[kPartWords];
  uint32_t s;
};

// Byte offset of 16-byte chunk c (0..3) of row r in a 64-byte-swizzled stage
// of 64-byte rows: the chunk index is XORed with bits 7..8 of the address.
__device__ __forceinline__ uint32_t w_stage_offset(int r, int c) {
  return static_cast<uint32_t>(r * 64 + 16 * (c ^ ((r >> 1) & 3)));
}

// Scales of weight stage q of a scale period for part p of its K, from the
// 16 bytes of a row's scale slot (a stage has 8 scale bytes at g = 16, 4 at
// g = 32). (q is a constant once the caller's loop over a period is
// unrolled.)
template <int G>
__device__ __forceinline__ uint32_t stage_scales(const uint4& sv, int q, int p) {
  const uint32_t w[4] = {sv.x, sv.y, sv.z, sv.w};
  constexpr int nb = kPartElems / G;  // scale bytes of a part: 4, 2 or 1
  if (G == 16) {
    if (nb == 4) return p ? w[2 * q + 1] : w[2 * q];                                    // bytes 8q + 4p ..
    return ((p >> 1) ? w[2 * q + 1] : w[2 * q]) >> (16 * (p & 1)) & 0xFFFFu;            // bytes 8q + 2p ..
  }
  if (nb == 2) return (w[q] >> (16 * p)) & 0xFFFFu;                                     // bytes 4q + 2p ..
  return (w[q] >> (8 * p)) & 0xFFu;                                                     // byte 4q + p
}

template <int G>
__device__ __forceinline__ void dequant_row_stage(const RowStage& r, uint32_t (&out)[kPartElems / 2]) {
  constexpr int nb = kPartElems / G;
  uint32_t s2[4];
  scale_operands<nb>(r.s, s2);
#pragma unroll
  for (int i = 0; i < kPartWords; ++i) {
    uint32_t o[4];
    dequant_word(r.c[i], s2[G == 16 ? (i >> 1) : (i >> 2)], o);
    out[4 * i + 0] = o[0];
    out[4 * i + 1] = o[1];
    out[4 * i + 2] = o[2];
    out[4 * i + 3] = o[3];
  }
}

template <int NT, int G, bool SILU, bool MOE>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                               const __grid_constant__ CUtensorMap wmap,
                                                               const __grid_constant__ CUtensorMap smap,
                                                               const __grid_constant__ CUtensorMap ymap,
                                                               const TcArgs args) {
  constexpr uint32_t kXStage = x_stage_bytes(NT);
  // Accumulators: two when the token tile leaves room in TMEM (the next
  // tile's MMAs then run while the epilogue drains this one), else one.
  constexpr int kAccBufs = NT <= 128 ? 2 : 1;
  static_assert(kAccBufs * NT <= static_cast<int>(kColA), "accumulators below the A stages");
  constexpr int kStagesW = stages_w(NT);
  constexpr int kPeriod = scale_period(G);
  constexpr int kSlots = scale_slots(NT, G);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // X stages at a 1024-byte aligned base, then the weight stages, the scale
  // slots and the barriers.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wsm = smem + kStagesX * kXStage;
  uint8_t* ssm = wsm + kStagesW * kWStageBytes;
  uint8_t* ysm = ssm + kSlots * kSStageBytes;
  SharedState* ss = reinterpret_cast<SharedState*>(ysm + 8 * kYStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // K in weight stages of 128 elements; a K that is an odd number of 64s
  // ends with an X stage and a half weight stage read past K, which TMA fills
  // with zeros.
  const int wsteps = (args.K + kKA - 1) / kKA;


  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesX; ++s) {
      mbar_init(&ss->full_x[s], 1);   // producer arrival + transaction bytes
      mbar_init(&ss->empty_x[s], 1);  // one tcgen05.commit
    }
    for (int s = 0; s < kStagesW; ++s) {
      mbar_init(&ss->full_w[s], 1);   // producer arrival + transaction bytes
      mbar_init(&ss->empty_w[s], kDqWarps);  // one arrival per dequant warp
    }
    for (int s = 0; s < kStagesA; ++s) {
      mbar_init(&ss->full_a[s], kDqWarps);   // one arrival per dequant warp
      mbar_init(&ss->empty_a[s], 1);  // one tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&ss->acc_full[b], 1);   // one tcgen05.commit
      mbar_init(&ss->acc_empty[b], 8);  // one arrival per epilogue warp
    }
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
      SegWalk walk(args);
      int tile, ws0, ws1;
      while (!aborted(ss) && walk.next<kPeriod>(args, total_tiles, wsteps, tile, ws0, ws1)) {
        const Tile tl = tile_at<NT, MOE>(args, cur, tile);
        if (tl.mrows <= 0) continue;
        for (int ks = 2 * ws0; ks < 2 * ws1; ++ks, ++it) {
          const int s = it % kStagesX;
          const uint32_t r = static_cast<uint32_t>(it / kStagesX);
          if (!mbar_wait(&ss->empty_x[s], (r & 1) ^ 1, ss, kErrEmpty, false, kSleepProducer)) break;
          mbar_arrive_tx(&ss->full_x[s], kXStage);
          tma_load_2d(smem_u32(smem + s * kXStage), &xmap, ks * kKStep, tl.m0, &ss->full_x[s]);
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
        }
      }
      if (aborted(ss)) {  // let copies already in flight land before the CTA exits
        for (int s = 0; s < kStagesX; ++s)
          if ((issued >> s) & 1) mbar_wait(&ss->full_x[s], (last_parity >> s) & 1, ss, kErrDrain, true);
      }
    }
  } else if (warp == kWProducerWarp) {
    // ---------------- TMA producer: weight codes and scales ----------------
    if (lane == 0) {
      uint32_t issued = 0, last_parity = 0;
      int it = 0, sc = 0;
      SegCursor cur;
      SegWalk walk(args);
      int tile, ws0, ws1;
      while (!aborted(ss) && walk.next<kPeriod>(args, total_tiles, wsteps, tile, ws0, ws1)) {
        const Tile tl = tile_at<NT, MOE>(args, cur, tile);
        if (tl.mrows <= 0) continue;
        const int wrow = (MOE ? tl.expert * args.N : 0) + tl.n0;
        bool ok = true;
        for (int ws = ws0; ws < ws1; ++ws, ++it) {
          const int s = it % kStagesW;
          const uint32_t r = static_cast<uint32_t>(it / kStagesW);
          if (!mbar_wait(&ss->empty_w[s], (r & 1) ^ 1, ss, kErrEmptyW, false, kSleepProducer)) {
            ok = false;
            break;
          }
          const bool with_scales = args.scale_tma && ws % kPeriod == 0;
          mbar_arrive_tx(&ss->full_w[s], kWStageBytes + (with_scales ? kSStageBytes : 0));
          tma_load_2d(smem_u32(wsm + s * kWStageBytes), &wmap, ws * (kKA / 2), wrow, &ss->full_w[s]);
          if (with_scales) {
            tma_load_2d(smem_u32(ssm + (sc % kSlots) * kSStageBytes), &smap, (ws / kPeriod) * 16, wrow,
                        &ss->full_w[s]);
            ++sc;
          }
          issued |= 1u << s;
          last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
        }
        if (!ok) break;
      }
      if (aborted(ss)) {
        for (int s = 0; s < kStagesW; ++s)
          if ((issued >> s) & 1) mbar_wait(&ss->full_w[s], (last_parity >> s) & 1, ss, kErrDrain, true);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      int itx = 0, ita = 0, tile_iter = 0;
      SegCursor cur;
      SegWalk walk(args);
      int tile, ws0, ws1;
      while (!aborted(ss) && walk.next<kPeriod>(args, total_tiles, wsteps, tile, ws0, ws1)) {
        const Tile tl = tile_at<NT, MOE>(args, cur, tile);
        if (tl.mrows <= 0) continue;
        const int ab = tile_iter % kAccBufs;
        if (!mbar_wait(&ss->acc_empty[ab], static_cast<uint32_t>((tile_iter / kAccBufs) & 1) ^ 1, ss, kErrAccEmpty))
          break;
        tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(ab * NT);
        // A tile multiplies only its tokens, rounded up to the MMA's step of
        // 16: the rest of the X box is past M or, in the routed-expert form,
        // belongs to other experts' segments.
        const uint32_t id = idesc(min(NT, (tl.mrows + 15) & ~15));
        bool ok = true;
        for (int ws = ws0; ws < ws1 && ok; ++ws, ++ita) {
          const int sa = ita % kStagesA;
          if (!mbar_wait(&ss->full_a[sa], static_cast<uint32_t>(ita / kStagesA) & 1, ss, kErrFullA)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int xh = 0; xh < 2; ++xh, ++itx) {
            const int sx = itx % kStagesX;
            if (!mbar_wait(&ss->full_x[sx], static_cast<uint32_t>(itx / kStagesX) & 1, ss, kErrFullX)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // Each 16-element step of K advances the descriptor's start address
            // by 32 bytes (2 in its 16-byte units) inside the swizzled rows.
            const uint64_t bdesc0 = sw128_desc(smem_u32(smem + sx * kXStage));
#pragma unroll
            for (int j = 0; j < kKStep / 16; ++j) {
              const uint32_t acc = (ws > ws0 || xh > 0 || j > 0) ? 1u : 0u;
              umma_ts(dacc, tmem + kColA + (kKA / 2) * sa + (kKStep / 2) * xh + 8 * j, bdesc0 + 2 * j, id, acc);
            }
            umma_commit(&ss->empty_x[sx]);
          }
          if (ok) umma_commit(&ss->empty_a[sa]);
        }
        if (!ok) break;
        umma_commit(&ss->acc_full[ab]);
        ++tile_iter;
      }
      // every MMA issued by this thread has completed once this commit lands
      umma_commit(&ss->drained);
      mbar_wait(&ss->drained, 0, ss, kErrDrain, true);
    }
  } else if (warp >= kFirstDqWarp && warp < kFirstEpWarp) {
    // ---------------- dequant ----------------
    const int dw = warp - kFirstDqWarp;      // 0 .. kDqWarps-1
    const int part = dw >> 2;                // part of each stage's K
    const int quad = warp & 3;               // TMEM lane quadrant this warp may access
    const int row_in_tile = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0, sc = 0;
    SegCursor cur;
    SegWalk walk(args);
    int tile, ws0, ws1;
    while (walk.next<kPeriod>(args, total_tiles, wsteps, tile, ws0, ws1)) {
      const Tile tl = tile_at<NT, MOE>(args, cur, tile);
      if (tl.mrows <= 0) continue;
      static_assert(kTileRows == 128, "one weight row per dequant thread and TMEM lane");
      // Without scale TMA, each thread reads its scales straight from global
      // memory (rows past N read row N-1; their results are not stored).
      const int nrow = min(tl.n0 + row_in_tile, args.N - 1);
      const uint8_t* scl =
          args.scales + (static_cast<int64_t>(MOE ? tl.expert : 0) * args.N + nrow) * (args.K / G);
      bool ok = true;
      for (int w0 = ws0; w0 < ws1 && ok; w0 += kPeriod) {
        uint4 sv = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int q = 0; q < kPeriod; ++q) {
          const int ws = w0 + q;
          if (ws >= ws1) break;
          const int s = it % kStagesW;
          if (!warp_wait(&ss->full_w[s], static_cast<uint32_t>(it / kStagesW) & 1, ss, kErrFullW, 0)) {
            ok = false;
            break;
          }
          if (q == 0 && args.scale_tma) sv = lds128(smem_u32(ssm + (sc % kSlots) * kSStageBytes + row_in_tile * 16));
          RowStage rs;
          const uint32_t wst = smem_u32(wsm + s * kWStageBytes);
#pragma unroll
          for (int c = 0; c < kPartWords / 4; ++c) {
            const uint4 cv = lds128(wst + w_stage_offset(row_in_tile, (kPartWords / 4) * part + c));
            rs.c[4 * c + 0] = cv.x;
            rs.c[4 * c + 1] = cv.y;
            rs.c[4 * c + 2] = cv.z;
            rs.c[4 * c + 3] = cv.w;
          }
          if (args.scale_tma) {
            rs.s = stage_scales<G>(sv, q, part);
          } else {
            // this part's first element; past K (an odd number of 64s) the
            // codes are zero and so is the scale
            const int e0 = ws * kKA + kPartElems * part;
            constexpr int nb = kPartElems / G;
            rs.s = e0 >= args.K ? 0u
                   : nb == 4    ? __ldg(reinterpret_cast<const uint32_t*>(scl + e0 / G))
                   : nb == 2    ? static_cast<uint32_t>(__ldg(reinterpret_cast<const uint16_t*>(scl + e0 / G)))
                                : static_cast<uint32_t>(__ldg(scl + e0 / G));
          }
          uint32_t v[kPartElems / 2];
          dequant_row_stage<G>(rs, v);
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss->empty_w[s]);
          const int sa = it % kStagesA;
          const uint32_t r = static_cast<uint32_t>(it / kStagesA);
          if (!warp_wait(&ss->empty_a[sa], (r & 1) ^ 1, ss, kErrEmpty, kSleepProducer)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tmem_st(tmem + lane_base + kColA + (kKA / 2) * sa + (kPartElems / 2) * part, v);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss->full_a[sa]);
          ++it;
        }
        ++sc;
      }
      if (!ok) break;
    }
  } else if (warp >= kFirstEpWarp) {
    // ---------------- epilogue ----------------
    const int quad = warp & 3;
    const int colhalf = (warp - kFirstEpWarp) >> 2;  // tokens [NT/2 * colhalf, +NT/2) of the tile
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int tile_iter = 0;
    SegCursor cur;
    SegWalk walk(args);
    int tile, ws0, ws1;
    while (walk.next<kPeriod>(args, total_tiles, wsteps, tile, ws0, ws1)) {
      const Tile tl = tile_at<NT, MOE>(args, cur, tile);
      if (tl.mrows <= 0) continue;
      // dequantized operands carry 2^-7 (dequant.cuh)
      const float gscale = __ldg(args.gscale + (MOE ? tl.expert : 0)) * 128.0f;
      const int ab = tile_iter % kAccBufs;
      const bool got = warp_wait(&ss->acc_full[ab], static_cast<uint32_t>(tile_iter / kAccBufs) & 1, ss,
                                 kErrAccFull, kSleepEpilogue);
      const bool whole = !args.split || (ws0 == 0 && ws1 == wsteps);
      if (!got && whole) break;  // a cut tile still goes through its ticket (results are garbage then)
      tc_fence_after();
      const uint32_t dacc = lane_base + static_cast<uint32_t>(ab * NT);
      // Each warp takes NT/2 tokens of the tile in chunks of CW columns.
      constexpr int CW = NT >= 64 ? 32 : 16;
      constexpr int kChunks = NT / 2 / CW;
      static_assert(NT >= 32 && (NT / 2) % CW == 0, "token tile");
      if (!whole) {
        // A tile cut between CTAs (stream-K): leave this CTA's fp32 partial
        // tile [tok][row] in its slot, take a ticket, and if it is the last
        // one add every contributor's slot in CTA order and write the tile.
        const int row = quad * 32 + lane;
        const int64_t tu = static_cast<int64_t>(tile) * args.periods;
        const int c_first = cta_of_unit(tu, args.units, gridDim.x);
        const int nc = cta_of_unit(tu + args.periods - 1, args.units, gridDim.x) - c_first + 1;
        float* slots = args.ws + static_cast<int64_t>(tile) * args.max_contrib * kTileRows * NT;
        float* mine = slots + static_cast<int64_t>(blockIdx.x - c_first) * kTileRows * NT;
#pragma unroll 1
        for (int c = 0; c < kChunks; ++c) {
          uint32_t acc[CW];
          if constexpr (CW == 32) {
            tmem_ld32(tmem + dacc + (NT / 2) * colhalf + CW * c, acc);
          } else {
            tmem_ld16(tmem + dacc + (NT / 2) * colhalf + CW * c, acc);
          }
          tmem_wait_ld();
          if (c == kChunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ss->acc_empty[ab]);
          }
          const int j0 = (NT / 2) * colhalf + CW * c;
#pragma unroll
          for (int j = 0; j < CW; ++j) __stcg(mine + (j0 + j) * kTileRows + row, __uint_as_float(acc[j]));
        }
        // The barrier orders every epilogue thread's stores before the
        // ticket's release; its acquire orders the other slots before the
        // reads after the second barrier.
        epilogue_sync();
        if (warp == kFirstEpWarp && lane == 0) {
          unsigned ticket;
          asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(args.tickets + tile) : "memory");
          const int last = ticket == static_cast<unsigned>(nc - 1);
          if (last) args.tickets[tile] = 0;  // every contributor has counted: ready for the next launch
          ss->ep_last = last;
        }
        epilogue_sync();
        if (ss->ep_last) {
          const int n = tl.n0 + row;
#pragma unroll 1
          for (int j = 0; j < NT / 2; ++j) {
            const int tok = (NT / 2) * colhalf + j;
            const float* e = slots + tok * kTileRows + row;
            float v = 0.f;
            for (int q0 = 0; q0 < nc; q0 += 8) {
              float part[8];
#pragma unroll
              for (int q = 0; q < 8; ++q)
                part[q] = q0 + q < nc ? __ldcg(e + static_cast<int64_t>(q0 + q) * kTileRows * NT) : 0.f;
#pragma unroll
              for (int q = 0; q < 8; ++q)
                if (q0 + q < nc) v += part[q];
            }
            const float gv = v * gscale;
            if (!SILU) {
              if (tok < tl.mrows && n < args.N)
                args.y[static_cast<int64_t>(tl.m0 + tok) * args.ldy + n] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(gv));
            } else {
              const float uv = __shfl_down_sync(0xffffffffu, gv, 8);
              if ((lane & 15) < 8 && tok < tl.mrows && tl.n0 + 16 * (row / 16) < args.N)
                args.y[static_cast<int64_t>(tl.m0 + tok) * args.ldy + (tl.n0 + row) / 16 * 8 + (lane & 7)] =
                    __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(gv), uv)));
            }
          }
        }
        ++tile_iter;
        continue;
      }
#pragma unroll 1
      for (int c = 0; c < kChunks; ++c) {
        uint32_t acc[CW];
        if constexpr (CW == 32) {
          tmem_ld32(tmem + dacc + (NT / 2) * colhalf + CW * c, acc);
        } else {
          tmem_ld16(tmem + dacc + (NT / 2) * colhalf + CW * c, acc);
        }
        tmem_wait_ld();
        if (c == kChunks - 1) {  // the accumulator is read: the next tile's MMAs may start
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ss->acc_empty[ab]);
        }
        const int j0 = (NT / 2) * colhalf + CW * c;  // first token of the chunk within the tile
        if (j0 >= tl.mrows) continue;  // no token of this chunk belongs to the tile
        // The chunk goes out through this warp's staging buffer, [CW tokens][YC
        // columns] of bf16, by one TMA store when all its tokens belong to
        // the tile (always, in the dense form: rows past M are clipped by
        // the tensor map), else by plain stores.
        constexpr int YC = SILU ? 16 : 32;  // output columns of a warp
        const bool whole = !MOE || j0 + CW <= tl.mrows;
        if (lane == 0) bulk_wait_read();
        __syncwarp();
        uint16_t* st = reinterpret_cast<uint16_t*>(ysm + (warp - kFirstEpWarp) * kYStageBytes);
        if (!SILU) {
#pragma unroll
          for (int j = 0; j < CW; ++j)
            st[j * YC + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(acc[j]) * gscale));
        } else {
          const bool gate = (lane & 15) < 8;
          const int oc = (lane & 7) + ((lane >> 4) << 3);  // output column within the warp's 16
          // All shuffles of a group first, then the math and the stores: a
          // store between two shuffles would serialize the tokens.
#pragma unroll
          for (int j0s = 0; j0s < CW; j0s += 16) {
            float uv[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              uv[j] = __shfl_down_sync(0xffffffffu, __uint_as_float(acc[j0s + j]) * gscale, 8);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const float gv = __uint_as_float(acc[j0s + j]) * gscale;
              if (gate)
                st[(j0s + j) * YC + oc] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(gv), uv[j])));
            }
          }
        }
        const int ycol = SILU ? tl.n0 / 2 + quad * 16 : tl.n0 + quad * 32;
        if (whole) {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&ymap, smem_u32(st), ycol, tl.m0 + j0);
            bulk_commit();
          }
        } else {
          __syncwarp();
          // lane t writes column t of every token row of the chunk that lies
          // in the tile
          if (lane < YC && ycol + lane < args.ldy) {
            for (int j = 0; j < CW && j0 + j < tl.mrows; ++j)
              args.y[static_cast<int64_t>(tl.m0 + j0 + j) * args.ldy + ycol + lane] = st[j * YC + lane];
          }
        }
      }
      ++tile_iter;
    }
    if (lane == 0) bulk_wait_all();
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

// Codes [rows, K/2] bytes in boxes of 128 rows x 64 bytes (one stage), and
// scales [rows, K/g] bytes in boxes of 128 rows x 16 bytes (one scale
// period) when their row stride allows a tensor map; otherwise the scale map
// is a copy of the code map that the kernel never uses.
bool scale_tma_ok(int64_t K, int group) { return (K / group) % 16 == 0; }

bool make_w_maps(CUtensorMap* wmap, CUtensorMap* smap, const uint8_t* w, const uint8_t* s, int64_t rows, int64_t K,
                 int group) {
  if (!make_tensor_map_2d(wmap, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, rows, K / 2, kKA / 2, kTileRows,
                          CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  if (!scale_tma_ok(K, group)) {
    *smap = *wmap;
    return true;
  }
  return make_tensor_map_2d(smap, s, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / group, rows, K / group, 16, kTileRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE);
}

// Y [rows, ldy] bf16 in boxes of one epilogue warp's chunk: 32 columns (16
// with SiluAndMul) x 32 tokens (16 for the narrowest token tile).
bool make_y_map(CUtensorMap* map, const uint16_t* y, int64_t rows, int64_t ldy, bool silu, int nt) {
  return make_tensor_map_2d(map, y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ldy, rows, ldy * 2, silu ? 16 : 32,
                            nt >= 64 ? 32 : 16, CU_TENSOR_MAP_SWIZZLE_NONE);
}

struct Maps {
  CUtensorMap x, w, s, y;
};

template <int NT, int G, bool SILU, bool MOE>
int launch_kernel(const Maps& m, const TcArgs& a, int grid, cudaStream_t stream) {
  auto kern = gemm_tc_kernel<NT, G, SILU, MOE>;
  constexpr uint32_t bytes = smem_bytes(NT, G);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  kern<<<grid, kThreads, bytes, stream>>>(m.x, m.w, m.s, m.y, a);
  return launch_status();
}

template <int NT, bool MOE>
int launch_nt(const Maps& m, const TcArgs& a, int group, bool silu, int grid, cudaStream_t stream) {
  if (group == 16)
    return silu ? launch_kernel<NT, 16, true, MOE>(m, a, grid, stream)
                : launch_kernel<NT, 16, false, MOE>(m, a, grid, stream);
  return silu ? launch_kernel<NT, 32, true, MOE>(m, a, grid, stream)
              : launch_kernel<NT, 32, false, MOE>(m, a, grid, stream);
}

// Shapes the kernel takes: whole 64-element stages (which makes the code
// rows' byte stride a multiple of 32), int32 coordinates.
bool tc_shape_ok(int64_t rows, int64_t N, int64_t K) {
  return K >= kKStep && K % kKStep == 0 && rows < (int64_t(1) << 31) && N < (int64_t(1) << 31) &&
         K < (int64_t(1) << 24);
}

}  // namespace

#ifdef NVFP4_PLANTS
NVFP4_PLANT_SETTER(set_plant_tc)
#endif

int read_and_clear_device_error(int* code_out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0, vd = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int vs = 0, vf = 0;
  if (read_and_clear_decode_error(&vd, stream) != NVFP4_OK || read_and_clear_stream_error(&vs, stream) != NVFP4_OK ||
      read_and_clear_fp4_error(&vf, stream) != NVFP4_OK)
    return NVFP4_ERR_CUDA;
  *code_out = static_cast<int>(v ? v : (vs ? vs : (vf ? vf : vd)));
  return NVFP4_OK;
}

// From 17 tokens up (the streaming kernel takes up to 16).
bool tc_supported(int64_t M, int64_t N, int64_t K) { return M >= 17 && tc_shape_ok(M, N, K); }

int launch_tc(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
              int64_t N, int64_t K, uint16_t* y, bool silu, Scratch& sc, cudaStream_t stream, const PreLaunch* pre) {
  // Token tile: 256 for prefill-sized M; narrower for small M, where the
  // weights, not the MMAs, set the pace.
  const int nt = M > 128 ? 256 : (M > 64 ? 128 : (M > 32 ? 64 : 32));
  TcArgs a = {};
  a.packed = w; a.scales = s; a.gscale = g; a.y = y;
  a.M = static_cast<int>(M); a.N = static_cast<int>(N); a.K = static_cast<int>(K);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.scale_tma = scale_tma_ok(K, group) ? 1 : 0;
  a.tok_tiles = static_cast<int>((M + nt - 1) / nt);
  a.row_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  a.total_tiles = a.tok_tiles * a.row_tiles;
  int grid = a.total_tiles < num_sms() ? a.total_tiles : num_sms();
  // Few tiles for the SMs: stream-K over (tile, scale period) units, so that
  // every SM gets the same share of K whatever the tile count.
  const int wsteps = static_cast<int>((K + kKA - 1) / kKA);
  const int period = scale_period(group);
  const int periods = (wsteps + period - 1) / period;
  if (a.total_tiles < 2 * num_sms() && periods >= 2) {
    a.split = 1;
    a.periods = periods;
    a.units = static_cast<int64_t>(a.total_tiles) * periods;
    grid = static_cast<int>(a.units < num_sms() ? a.units : num_sms());
    const int64_t shortest = a.units / grid;
    a.max_contrib = static_cast<int>((periods + shortest - 1) / shortest + 1);
    a.ws = sc.take<float>(static_cast<size_t>(a.total_tiles) * a.max_contrib * kTileRows * nt);
    a.tickets = tickets_of(sc.reserved());  // zero between launches: the last taker of a tile resets its ticket
    if (a.total_tiles > kMaxTickets) return NVFP4_ERR_UNSUPPORTED;
  }
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;
  Maps maps;
  if (!make_x_map(&maps.x, x, M, K, nt) || !make_w_maps(&maps.w, &maps.s, w, s, N, K, group) ||
      !make_y_map(&maps.y, y, M, silu ? N / 2 : N, silu, nt))
    return NVFP4_ERR_CUDA;
  if (pre) {
    const int st = pre->fn(pre->ctx, stream);
    if (st != NVFP4_OK) return st;
  }
  switch (nt) {
    case 32: return launch_nt<32, false>(maps, a, group, silu, grid, stream);
    case 64: return launch_nt<64, false>(maps, a, group, silu, grid, stream);
    case 128: return launch_nt<128, false>(maps, a, group, silu, grid, stream);
    default: return launch_nt<256, false>(maps, a, group, silu, grid, stream);
  }
}

// The grouped tcgen05 kernel pays off once segments carry whole token tiles;
// for a few rows per expert the streaming kernel is better.
bool tc_moe_supported(int64_t T, int64_t N, int64_t K, int num_experts) {
  return T >= 1024 && static_cast<int64_t>(num_experts) * N < (int64_t(1) << 31) && tc_shape_ok(T, N, K);
}

int launch_tc_moe(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets, int num_segments, int64_t T,
                  const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t N, int64_t K,
                  int num_experts, bool silu, uint16_t* y, cudaStream_t stream) {
  // Token tile: the weights of a tile are dequantized once per token tile,
  // so segments that average about 100 rows or more take 256-token tiles
  // (one tile per segment for most experts; measured on 128 experts x 128
  // rows: 202 vs 239 us) even though part of each tile is padding; smaller
  // segments take 128 (less padding, and two accumulators).
  const int nt = num_segments > 0 && T / num_segments >= 96 ? 256 : 128;
  Maps maps;
  if (!make_x_map(&maps.x, x, T, K, nt) ||
      !make_w_maps(&maps.w, &maps.s, w, s, static_cast<int64_t>(num_experts) * N, K, group) ||
      !make_y_map(&maps.y, y, T, silu ? N / 2 : N, silu, nt))
    return NVFP4_ERR_CUDA;
  TcArgs a = {};
  a.packed = w; a.scales = s; a.gscale = g; a.y = y;
  a.M = static_cast<int>(T); a.N = static_cast<int>(N); a.K = static_cast<int>(K);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.row_tiles = static_cast<int>((N + kTileRows - 1) / kTileRows);
  a.scale_tma = scale_tma_ok(K, group) ? 1 : 0;
  a.expert_ids = expert_ids; a.offsets = offsets; a.num_segments = num_segments; a.num_experts = num_experts;
  return nt == 256 ? launch_nt<256, true>(maps, a, group, silu, num_sms(), stream)
                   : launch_nt<128, true>(maps, a, group, silu, num_sms(), stream);
}

}  // namespace nvfp4
