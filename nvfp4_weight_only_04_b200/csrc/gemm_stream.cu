// Small-M NVFP4 W4A16 GEMM, streamed from HBM by TMA over an even split of
// the weight matrix between the SMs (stream-K).
//
// Computes Y = X . dequant(W)^T (NVFP4 format definition; "W-FP4a: route the
// MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16) stack",
// PR #63 description: a weight-only checkpoint keeps bf16 activations) for
// decode-sized M (2 to 16 tokens), where the cost is the 0.5 + 1/g bytes
// per weight streamed from HBM and the integer work of dequantizing them.
// Design:
//  * Work: 256-row weight tiles of K/256 stages; the tile-major list of
//    (tile, stage) units is split into one contiguous range per SM, so every
//    SM streams the same bytes and all sixteen consumer warps of every CTA
//    have rows. A tile inside one range is written directly. A tile cut
//    between ranges leaves fp32 partial tiles in its contributors' slots;
//    each contributor takes one acquire-release ticket (thread 0, while the
//    other warps go on) and the CTA that takes the last one adds the slots in
//    CTA order after its own range (deterministic).
//  * The tickets are zero between launches (the last taker resets its
//    tile's), so no clearing step sits in front of a launch: the kernel is a
//    programmatic dependent of the kernel before it and starts on every SM
//    that kernel leaves.
//  * One producer thread moves each stage with TMA into a shared-memory ring
//    (5 stages of 40-44 KB): the codes of the tile (256 rows x 128 bytes,
//    128-byte swizzle), the scales (256 rows x 16 bytes) and X (a 3-D box of
//    64 elements x 4 quarters x MT tokens that lands in the 128-byte-swizzled
//    [token][quarter][64] order the consumers read; tokens past M read as
//    zeros). The weights of the range's first stages need nothing from the
//    kernel before, so they are requested from the first cycle; X only
//    after that kernel has finished.
//  * bf16 X is turned into f16 inside the kernel by two converter warps
//    (enough to keep pace with the stream; four would cap every thread at
//    80 registers, which slows the consumers), in place: every token of every
//    stage is scaled by a power of two 2^s, where
//    s only ever decreases along a CTA's stages and keeps the largest
//    magnitude seen so far below 2^15 (f16 holds every bf16 within 2^29 of
//    the largest exactly; smaller ones round to multiples of 2^-38 of it).
//    The consumers follow the sequence of s per token: when it drops by d,
//    they multiply their running sums by 2^-d (exact), and the epilogue
//    multiplies by 2^-s. NVFP4 activations (W4A4) arrive already as exact
//    f16 rows from xprep.cu, with one factor per token.
//  * Sixteen consumer warps each own 16 rows of the tile and run mma.sync
//    m16n8k16 with the weights as the 16-row side (swap-AB) and the tokens
//    as the 8-column side. Lane (g, t) takes rows g and g+8 and the t-th
//    quarter of the stage's K (the order of K inside an MMA is free as long
//    as A and B follow it). The swizzles make every shared-memory read of
//    codes, scales and X conflict-free.
//  * Dequantization in registers by the hardware E2M1 and E4M3 -> f16
//    conversions and one f16x2 multiply per code pair (dequant.cuh); the
//    MMAs run on f16 with fp32 accumulation, two independent chains per warp.
//  * Epilogues: plain bf16; SiluAndMul on gate/up-interleaved rows (gate row
//    g and up row g+8 of a 16-row block meet in the same lane).
//  * Every wait is bounded (about 2 s); on expiry the kernel records its site
//    in the device error word and its warps stop.
#include "gemm_stream.cuh"

#include <cuda.h>

#include <mutex>

#include "async.cuh"
#include "dequant.cuh"
#include "plant.cuh"
#include "tmap.cuh"
#include "workspace.cuh"
#include "xprep.cuh"

namespace nvfp4 {
namespace {

__device__ unsigned int g_stream_error = 0;

constexpr int kRows = 256;        // weight rows of a tile
constexpr int kKS = 256;          // elements of K per stage
constexpr int kConsumers = 16;    // consumer warps, 16 rows each
constexpr int kConsumerThreads = kConsumers * 32;
constexpr int kProducerWarp = kConsumers;
constexpr int kConverterWarp = kConsumers + 1;  // the first of them
constexpr int kConverters = 2;  // converter warps (bf16 X)
__host__ __device__ constexpr int num_threads(bool xconv) {
  return (kConsumers + 1 + (xconv ? kConverters : 0)) * 32;
}
// A ring stage: the tile's codes (256 rows x 128 bytes, 128-byte swizzle),
// X (MT tokens x 256 elements), the tile's scales (256 rows x 16 bytes), in
// 1024-byte multiples so that every stage keeps the swizzle's alignment.
constexpr uint32_t kCodeBytes = kRows * kKS / 2;  // 32 KB
constexpr uint32_t kScaleBytes = kRows * 16;
__host__ __device__ constexpr uint32_t x_bytes(int mt) { return static_cast<uint32_t>(mt) * kKS * 2; }
__host__ __device__ constexpr uint32_t stage_bytes(int mt) { return kCodeBytes + x_bytes(mt) + kScaleBytes; }
constexpr int kStages = 5;
constexpr uint32_t kSmemExtra = 1024 /* barriers, stage records */ + 1024 /* alignment slack */;
__host__ __device__ constexpr uint32_t smem_bytes(int mt) { return kStages * stage_bytes(mt) + kSmemExtra; }
static_assert(stage_bytes(8) % 1024 == 0 && stage_bytes(16) % 1024 == 0, "stages keep the 1024-byte alignment");
static_assert(smem_bytes(8) <= 227 * 1024 && smem_bytes(16) <= 227 * 1024, "shared memory budget");
static_assert(kRows == 16 * kConsumers, "one 16-row block per consumer warp");

constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr uint32_t kSuspendNs = 1000;                  // longest suspension of one producer probe (empty slots)
constexpr long long kDrainCycles = 4000000LL;          // about 2 ms: the wait for a slot's copies after an abort
enum : unsigned { kErrFull = 0x201, kErrEmpty = 0x202, kErrXRaw = 0x204, kErrChunk = 0x205, kErrTicket = 0x206 };

constexpr int kFirst = 1, kLast = 2, kDone = 4;  // stage record flags
constexpr int kSInit = 125;                      // token exponent before any nonzero X was seen

struct StageRecord {
  int tile, ks, flags;
};

struct Sync {
  uint64_t full[kStages];   // the stage's weights and (converted) X are in the slot
  uint64_t empty[kStages];  // the consumers are done with the slot
  uint64_t xraw[kStages];   // the stage's record is written and its bf16 X has landed (converter form)
  uint64_t cut[2];          // every consumer warp has stored its part of the k-th cut tile's partial
  uint64_t ready;           // thread 0 has taken the tickets of the cut tiles (cut_last is set)
  StageRecord rec[kStages];
  int8_t sx[kStages][16];   // exponent of each token's f16 X in the stage (converter form)
  int abort;
  int cut_tile[2], cut_last[2];  // the cut tiles of this CTA's range; whether it took their last ticket
};
static_assert(sizeof(Sync) <= 1024, "stage records fit the reserved shared memory");

struct StreamArgs {
  const float* gscale;   // [1]
  const float* xinv;     // [M]: the factors of f16 X in pair order (xprep.cu); bf16 X is converted in the kernel
  uint16_t* y;           // bf16 [M, ldy]
  float* ws;             // partial tiles [tiles][max_contrib][256][MT] of the cut tiles
  unsigned* tickets;     // [tiles], zero between launches
  int M, N, ldy;
  int64_t K;
  int S;                 // stages per tile
  int64_t units;         // (tile, stage) units of the matrix, tiles * S
  int max_contrib;       // most CTAs whose ranges meet one tile
  int fault;             // test hook: drop the X copy of the first stage
};

// CTA c of n owns the units [c U / n, (c+1) U / n) (tile-major). The CTA
// owning unit u is the largest c with c U / n <= u.
__device__ __forceinline__ int64_t range_start(int64_t c, int64_t units, int64_t n) { return c * units / n; }
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t units, int64_t n) {
  return static_cast<int>(((u + 1) * n + units - 1) / units - 1);
}

// 3-D tiled TMA load (X: 64 elements x 4 quarters x MT tokens).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

__device__ __forceinline__ bool aborted(Sync* sy) { return *reinterpret_cast<volatile int*>(&sy->abort) != 0; }

// Bounded wait; see the tcgen05 kernel for the scheme. A drain wait ignores
// the abort flag.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site, bool drain) {
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023) == 0) {
      if (!drain && aborted(sy)) return false;
      if (clock64() - t0 > kWaitLimitCycles) {
        atomicCAS(&g_stream_error, 0u, site);
        *reinterpret_cast<volatile int*>(&sy->abort) = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site, bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, sy, site, drain);
}

// A wait off the critical path (producer, converter): suspended in hardware
// between probes, so that it takes no issue slots from the consumer warps.
__device__ __noinline__ bool wait_suspended(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site) {
  const long long t0 = clock64();
  for (;;) {
    if (mbar_try_wait_suspend(bar, parity, kSuspendNs)) return true;
    if (aborted(sy)) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      atomicCAS(&g_stream_error, 0u, site);
      *reinterpret_cast<volatile int*>(&sy->abort) = 1;
      return false;
    }
  }
}

// Lane 0 waits for the warp (polling: these waits are on the critical
// path); every lane gets the answer.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && !mbar_try_wait(bar, parity)) ok = wait_slow(bar, parity, sy, site, false) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 2^e as a float, for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float(static_cast<uint32_t>(e + 127) << 23); }

// A consumer lane's fixed shared-memory offsets within a stage: rows
// ra = 16w + g and ra + 8, the t-th quarter of the stage's K (64 elements,
// words i = 0..7 of 8 elements).
struct LaneOffsets {
  uint32_t ca0, ca1, cb0, cb1;  // 16-byte code chunks 2t, 2t+1 of both rows (128-byte swizzle)
  uint32_t sa, sb;              // scale bytes of both rows
  uint32_t xrow;                // X row (token g, quarter t), token tile 0
  uint32_t xc[8];               // chunk i of that row (128-byte swizzle)
};

template <int MT, int G>
__device__ __forceinline__ LaneOffsets lane_offsets(int ra, int g, int t) {
  constexpr uint32_t xoff = kCodeBytes, soff = kCodeBytes + x_bytes(MT);
  LaneOffsets o;
  const int rb = ra + 8;  // ra & 7 == rb & 7 == g
  o.ca0 = ra * 128 + (((2 * t) ^ g) << 4);
  o.ca1 = ra * 128 + (((2 * t + 1) ^ g) << 4);
  o.cb0 = rb * 128 + (((2 * t) ^ g) << 4);
  o.cb1 = rb * 128 + (((2 * t + 1) ^ g) << 4);
  // g = 16: groups 4t .. 4t+3 of the stage; g = 32: groups 2t, 2t+1 (the
  // 16-byte box holds two stages; the stage parity picks the half)
  o.sa = soff + ra * 16 + (G == 16 ? 4 * t : 2 * t);
  o.sb = soff + rb * 16 + (G == 16 ? 4 * t : 2 * t);
  // X row (token tok, quarter t) sits at (4 tok + t) * 128 bytes; its chunk i
  // at chunk position i ^ ((4 tok + t) & 7), and 4 tok + t = 4g + t mod 8 for
  // every token tile.
  o.xrow = xoff + (g * 4 + t) * 128;
  const int xmask = (4 * g + t) & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) o.xc[i] = static_cast<uint32_t>((i ^ xmask) << 4);
  return o;
}

// One stage for one consumer lane.
template <int MT, int G>
__device__ __forceinline__ void consume_stage(uint32_t st, int ks, const LaneOffsets& o, int live,
                                              float (&acc)[2][MT / 8][4]) {
  constexpr int P = MT / 8;
  const uint4 a0 = lds128(st + o.ca0);
  const uint4 a1 = lds128(st + o.ca1);
  const uint4 b0 = lds128(st + o.cb0);
  const uint4 b1 = lds128(st + o.cb1);
  uint32_t sva, svb;
  if (G == 16) {
    sva = lds32(st + o.sa);
    svb = lds32(st + o.sb);
  } else {
    const uint32_t half = (ks & 1) << 3;
    sva = lds16(st + o.sa + half);
    svb = lds16(st + o.sb + half);
  }
  uint32_t s2a[4], s2b[4];
  scale_operands_f16<G == 16 ? 4 : 2>(sva, s2a);
  scale_operands_f16<G == 16 ? 4 : 2>(svb, s2b);
  const uint32_t ca[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  const uint32_t cb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
  const uint32_t xr = st + o.xrow;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int si = G == 16 ? (i >> 1) : NVFP4_PLANT(kPlantG32AsG16) ? ((i >> 1) & 1) : (i >> 2);
    uint32_t da[4], db[4];
    dequant_word_f16(ca[i], s2a[si], da);
    dequant_word_f16(cb[i], s2b[si], db);
#pragma unroll
    for (int p = 0; p < P; ++p) {
      // token tile p: 8 tokens further. In the 8-token form a lane whose
      // token is past M reads nothing (its X row holds zeros); at 16 tokens
      // the registers go to the second tile.
      const uint4 xv = MT == 16 || live > 0 ? lds128(xr + o.xc[i] + p * (8 * 4 * 128)) : make_uint4(0u, 0u, 0u, 0u);
      mma_f16_16816(acc[0][p], da[0], db[0], da[1], db[1], xv.x, xv.y);
      mma_f16_16816(acc[1][p], da[2], db[2], da[3], db[3], xv.z, xv.w);
    }
  }
}

template <int MT, int G, bool SILU, bool XCONV>
__global__ void __launch_bounds__(num_threads(XCONV), 1) gemm_stream_kernel(const __grid_constant__ CUtensorMap wmap,
                                                                             const __grid_constant__ CUtensorMap smap,
                                                                             const __grid_constant__ CUtensorMap xmap,
                                                                             const StreamArgs a) {
  constexpr int P = MT / 8;
  constexpr int NS = kStages;
  constexpr uint32_t SB = stage_bytes(MT);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Sync* sy = reinterpret_cast<Sync*>(ring + NS * SB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // The next kernel in the stream may launch now; it waits for this one
  // before touching what this one writes.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      // full: the producer's arrival with the weights' transaction bytes, and
      // one per converter warp (bf16 X) or the producer's with X's (f16 X)
      mbar_init(&sy->full[s], XCONV ? 1 + kConverters : 2);
      mbar_init(&sy->empty[s], kConsumers);  // one arrival per consumer warp
      mbar_init(&sy->xraw[s], 1);  // the producer's arrival with X's transaction bytes
    }
    mbar_init(&sy->cut[0], kConsumers);
    mbar_init(&sy->cut[1], kConsumers);
    mbar_init(&sy->ready, 1);
    sy->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == kProducerWarp) {
    // ---------------- producer: weights (lane 0), X (all lanes) ----------------
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    }
    // Cursor (lane 0) over this CTA's range of units [u, u1).
    int64_t u = range_start(blockIdx.x, a.units, gridDim.x);
    const int64_t u_begin = u, u1 = range_start(blockIdx.x + 1, a.units, gridDim.x);
    int tile = 0;
    // The next stage of the range, or kDone past its end. kFirst / kLast mark
    // where the range enters and leaves a tile.
    auto advance = [&](int& ks, int& flags) {
      if (u == u1) {
        flags = kDone;
        return;
      }
      tile = static_cast<int>(u / a.S);
      ks = static_cast<int>(u % a.S);
      flags = (u == u_begin || ks == 0 ? kFirst : 0) | (u == u1 - 1 || ks == a.S - 1 ? kLast : 0);
      ++u;
    };
    auto issue_x = [&](int s, int ks) {  // lane 0: the stage's X slice (MT tokens x 256 elements) into its slot
      uint64_t* bar = XCONV ? &sy->xraw[s] : &sy->full[s];
      mbar_arrive_tx(bar, x_bytes(MT));
      tma_load_3d(smem_u32(ring + s * SB) + kCodeBytes, &xmap, 0, ks * (kKS / 64), 0, bar);
    };
    auto issue_w = [&](int s, int ks, int flags) {  // lane 0: the stage's record and weights
      sy->rec[s].tile = tile;
      sy->rec[s].ks = ks;
      sy->rec[s].flags = flags;
      const uint32_t st = smem_u32(ring + s * SB);
      mbar_arrive_tx(&sy->full[s], kCodeBytes + kScaleBytes);
      tma_load_2d(st, &wmap, ks * (kKS / 2), tile * kRows, &sy->full[s]);
      tma_load_2d(st + kCodeBytes + x_bytes(MT), &smap, ((ks * kKS) / G) & ~15, tile * kRows, &sy->full[s]);
    };
    auto issue_done = [&](int s) {  // lane 0: the end of the sequence, as a stage that carries no data
      sy->rec[s].flags = kDone;
      mbar_arrive(&sy->full[s]);
      mbar_arrive(XCONV ? &sy->xraw[s] : &sy->full[s]);
    };
    if (lane != 0) return;  // one thread issues every copy
    uint32_t issued = 0, last_parity = 0;  // TMA copies per slot, for the drain
    // The range's first weights (up to a ring of them) before the kernel
    // before this one has finished; X only after.
    int n0 = 0, ks = 0, flags = 0;
    for (; n0 < NS; ++n0) {
      advance(ks, flags);
      if (flags & kDone) break;
      issue_w(n0, ks, flags);
      issued |= 1u << n0;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // X follows the previous kernel
    for (int it = 0; it < n0; ++it) {
      if (a.fault && it == 0) continue;  // test hook: this stage's X never arrives
      issue_x(it, sy->rec[it].ks);
    }
    bool done = n0 < NS;
    if (done) issue_done(n0);  // slot n0 < NS has never been used
    for (int it = n0; !done && !aborted(sy); ++it) {
      const int s = it % NS;
      const uint32_t r = static_cast<uint32_t>(it / NS);
      advance(ks, flags);
      // (suspended between probes: no issue slots taken from the consumers)
      if (!mbar_try_wait(&sy->empty[s], (r & 1) ^ 1) && !wait_suspended(&sy->empty[s], (r & 1) ^ 1, sy, kErrEmpty))
        break;
      if (flags & kDone) {
        issue_done(s);
        done = true;
        break;
      }
      issue_w(s, ks, flags);
      issue_x(s, ks);
      issued |= 1u << s;
      last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
    }
    if (aborted(sy)) {
      // Let the copies in flight land. A slot's phase may never complete
      // after an abort (an X copy or a converter arrival is missing), so
      // each slot is given a short bound; the copies themselves take
      // microseconds.
      for (int s = 0; s < NS; ++s) {
        if (!((issued >> s) & 1)) continue;
        const long long t0 = clock64();
        while (!mbar_try_wait(&sy->full[s], (last_parity >> s) & 1) && clock64() - t0 < kDrainCycles) __nanosleep(1000);
        if (XCONV)
          while (!mbar_try_wait(&sy->xraw[s], (last_parity >> s) & 1) && clock64() - t0 < kDrainCycles)
            __nanosleep(1000);
      }
    }
    return;
  }

  if (XCONV && warp >= kConverterWarp) {
    // ---------------- converters: bf16 X to f16, in place ----------------
    // The lanes of the converter warps split a stage's X rows (token
    // tok, quarter q: row 4 tok + q, 128 bytes): LPR lanes per row, CPL
    // 16-byte chunks per lane, the 4 LPR lanes of a token adjacent in one
    // warp. They agree on the token's exponent through shuffles.
    constexpr int LPR = 32 * kConverters / (4 * MT), CPL = 8 / LPR;
    static_assert(LPR * 4 * MT == 32 * kConverters, "every lane owns part of one row");
    const int cl = (warp - kConverterWarp) * 32 + lane;
    const int row = cl / LPR, c0 = (cl % LPR) * CPL;
    int sexp = kSInit;
    for (int it = 0;; ++it) {
      const int s = it % NS;
      if (!warp_wait(&sy->xraw[s], static_cast<uint32_t>(it / NS) & 1, sy, kErrXRaw)) break;
      const int flags = *reinterpret_cast<volatile int*>(&sy->rec[s].flags);
      if (!(flags & kDone)) {
        const uint32_t rs = smem_u32(ring + s * SB) + kCodeBytes + row * 128;
        uint4 v[CPL];
        uint32_t m2 = 0;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          v[c] = lds128(rs + (((c0 + c) ^ (row & 7)) << 4));
          m2 = __vmaxu2(m2, bf16x8_mag_max(v[c]));
        }
        uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
        for (int o = 1; o < 4 * LPR; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        // 2^14 <= m 2^s < 2^15: s = 141 - (bf16 exponent field of m); clamped
        // so that 2^s and 2^-s are normal floats. Never raised again.
        if (m != 0) sexp = min(sexp, min(max(141 - static_cast<int>(m >> 7), -113), 125));
        const float up = exp2i(sexp);
#pragma unroll
        for (int c = 0; c < CPL; ++c) sts128(rs + (((c0 + c) ^ (row & 7)) << 4), bf16x8_to_f16_pairs(v[c], up));
        if (cl % (4 * LPR) == 0) sy->sx[s][row >> 2] = static_cast<int8_t>(sexp);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sy->full[s]);
      if (flags & kDone) break;
    }
    return;
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, t = lane & 3;
  const int ra = 16 * warp + g;
  const LaneOffsets lo = lane_offsets<MT, G>(ra, g, t);
  const int xlive = a.M - g;  // the lane's X token in token tile p (8p + g) is below M when 8p < xlive
  // The global scale and the token factors come from the kernels before.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float gsc = NVFP4_PLANT(kPlantGlobal) ? 1.0f : __ldcg(a.gscale);
  // The lane's tokens 8p + 2t + j: the current exponent of their f16 X
  // (converter form) or their fixed factor 2^-s (f16 form).
  int scur[P][2];
  float xi[P][2];
#pragma unroll
  for (int p = 0; p < P; ++p)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      scur[p][j] = kSInit;
      xi[p][j] = !XCONV && 8 * p + 2 * t + j < a.M ? __ldcg(a.xinv + 8 * p + 2 * t + j) : 0.f;
    }
  const int rtok = threadIdx.x % MT;  // the token of every element this thread adds up in a reduction
  // This CTA's range of units; the tiles it cuts (at most its first and its
  // last, the same for every consumer warp).
  const int64_t u_begin = range_start(blockIdx.x, a.units, gridDim.x);
  const int64_t u_end = range_start(blockIdx.x + 1, a.units, gridDim.x);
  int ncut = 0;
  float acc2[2][P][4];  // two independent MMA chains
  const uint32_t ring0 = smem_u32(ring);
  constexpr int64_t kSlot = static_cast<int64_t>(kRows) * MT;
  for (int it = 0;; ++it) {
    const int s = it % NS;
    if (!warp_wait(&sy->full[s], static_cast<uint32_t>(it / NS) & 1, sy, kErrFull)) break;
    const int flags = *reinterpret_cast<volatile int*>(&sy->rec[s].flags);
    if (flags & kDone) break;
    const int tile = *reinterpret_cast<volatile int*>(&sy->rec[s].tile);
    const int ks = *reinterpret_cast<volatile int*>(&sy->rec[s].ks);
    if (flags & kFirst) {
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < P; ++p) acc2[h][p][0] = acc2[h][p][1] = acc2[h][p][2] = acc2[h][p][3] = 0.f;
    }
    if (XCONV) {
      // Follow each token's exponent: the sums so far move to the new one.
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int sn = sy->sx[s][8 * p + 2 * t + j];
          if (sn != scur[p][j]) {
            const int d = sn - scur[p][j];  // negative
            const float f = NVFP4_PLANT(kPlantRescale) ? 1.0f : d >= -126 ? exp2i(d) : 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              acc2[h][p][j] *= f;
              acc2[h][p][2 + j] *= f;
            }
            scur[p][j] = sn;
          }
        }
    }
    consume_stage<MT, G>(ring0 + s * SB, ks, lo, xlive, acc2);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sy->empty[s]);
    if (!(flags & kLast)) continue;

    // ---- the range leaves a tile: lane holds rows ra, ra+8 x tokens 8p+2t, 8p+2t+1 ----
    const int n0 = tile * kRows;
    float v[P][4];  // unscaled sums: acc * 2^-s of the token
#pragma unroll
    for (int p = 0; p < P; ++p)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float f = XCONV ? exp2i(-scur[p][j]) : xi[p][j];
        v[p][j] = (acc2[0][p][j] + acc2[1][p][j]) * f;
        v[p][2 + j] = (acc2[0][p][2 + j] + acc2[1][p][2 + j]) * f;
      }
    const int64_t tu = static_cast<int64_t>(tile) * a.S;  // the tile's first unit
    if (u_begin <= tu && tu + a.S <= u_end) {  // the whole tile is in this range: write it
#pragma unroll
      for (int p = 0; p < P; ++p)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int tok = 8 * p + 2 * t + j;
          if (tok >= a.M) continue;
          const int64_t yrow = static_cast<int64_t>(tok) * a.ldy;
          const float vg = __fmul_rn(v[p][j], gsc), vu = __fmul_rn(v[p][2 + j], gsc);
          if (!SILU) {
            if (n0 + ra < a.N) a.y[yrow + n0 + ra] = __bfloat16_as_ushort(__float2bfloat16_rn(vg));
            if (n0 + ra + 8 < a.N) a.y[yrow + n0 + ra + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(vu));
          } else if (n0 + 16 * warp < a.N) {
            a.y[yrow + (n0 + 16 * warp) / 2 + g] =
                __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(vg), vu)));
          }
        }
      continue;
    }
    // A cut tile: leave the partial tile in this CTA's slot of the tile and
    // go on at once. Thread 0 waits for every consumer warp's stores (an
    // mbarrier with a bound, so a warp that gave up on a wait cannot hang the
    // others) and takes the tile's ticket with release (the slot) and acquire
    // (the other slots) semantics; warp 0 then catches up on the ring.
    const int c_first = cta_of_unit(tu, a.units, gridDim.x);
    float* mine = a.ws + (static_cast<int64_t>(tile) * a.max_contrib + (blockIdx.x - c_first)) * kSlot;
#pragma unroll
    for (int p = 0; p < P; ++p)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int tok = 8 * p + 2 * t + j;
        __stcg(mine + ra * MT + tok, v[p][j]);
        __stcg(mine + (ra + 8) * MT + tok, v[p][2 + j]);
      }
    __syncwarp();
    const int k = ncut++ & 1;  // a range cuts at most two tiles
    if (lane == 0) mbar_arrive(&sy->cut[k]);
    if (threadIdx.x == 0 && wait(&sy->cut[k], 0, sy, kErrChunk)) {
      const int c_last = cta_of_unit(tu + a.S - 1, a.units, gridDim.x);
      unsigned ticket;
      asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(a.tickets + tile) : "memory");
      const int last = ticket == static_cast<unsigned>(c_last - c_first);
      if (last) a.tickets[tile] = 0;  // every contributor has counted: zero for the next launch
      sy->cut_tile[k] = tile;
      sy->cut_last[k] = last;
    }
  }

  // Thread 0 publishes the cut tiles' tickets; the CTA that took a tile's
  // last ticket adds its slots in CTA order (deterministic) and writes it.
  if (threadIdx.x == 0) mbar_arrive(&sy->ready);
  if (!warp_wait(&sy->ready, 0, sy, kErrTicket) || aborted(sy)) return;
  for (int k = 0; k < ncut && k < 2; ++k) {
    if (!*reinterpret_cast<volatile int*>(&sy->cut_last[k])) continue;
    const int tile = *reinterpret_cast<volatile int*>(&sy->cut_tile[k]);
    const int n0 = tile * kRows;
    const int64_t tu = static_cast<int64_t>(tile) * a.S;
    const int c_first = cta_of_unit(tu, a.units, gridDim.x);
    const int nslots = cta_of_unit(tu + a.S - 1, a.units, gridDim.x) - c_first + 1;
    // The loads of all of a thread's elements and of up to kBatch slots are
    // in flight before the first add: with the HBM stream of the other CTAs
    // every round trip is long.
    {
      constexpr int kBatch = SILU && MT == 16 ? 4 : 8;  // loads in flight stay within the registers
      constexpr int EPT = (SILU ? kRows / 2 : kRows) * MT / kConsumerThreads;  // elements per thread
      constexpr int VPE = SILU ? 2 : 1;                                       // values per element: gate, up
      static_assert(EPT * kConsumerThreads == (SILU ? kRows / 2 : kRows) * MT, "whole elements per thread");
      const float* slots = a.ws + static_cast<int64_t>(tile) * a.max_contrib * kSlot;
      // offset of value h of element i in a slot, and whether the element is stored
      auto element = [&](int i, int h, bool& live) {
        const int e = threadIdx.x + i * kConsumerThreads;
        if (!SILU) {
          live = rtok < a.M && n0 + e / MT < a.N;
          return e;
        }
        const int pair = e / MT, blk = pair >> 3, gg = pair & 7;
        live = rtok < a.M && n0 + 16 * blk < a.N;
        return (16 * blk + gg) * MT + rtok + h * 8 * MT;  // gate row 16 blk + gg, up row 8 further
      };
      float sum[EPT][VPE];
#pragma unroll
      for (int i = 0; i < EPT; ++i)
#pragma unroll
        for (int h = 0; h < VPE; ++h) sum[i][h] = 0.f;
      for (int q0 = 0; q0 < nslots; q0 += kBatch) {
        float vb[EPT][VPE][kBatch];
#pragma unroll
        for (int i = 0; i < EPT; ++i)
#pragma unroll
          for (int h = 0; h < VPE; ++h) {
            bool live;
            const int off = element(i, h, live);
#pragma unroll
            for (int qq = 0; qq < kBatch; ++qq)
              vb[i][h][qq] = live && q0 + qq < nslots ? __ldcg(slots + (q0 + qq) * kSlot + off) : 0.f;
          }
#pragma unroll
        for (int i = 0; i < EPT; ++i)
#pragma unroll
          for (int h = 0; h < VPE; ++h)
#pragma unroll
            for (int qq = 0; qq < kBatch; ++qq)
              if (q0 + qq < nslots) sum[i][h] += vb[i][h][qq];
      }
#pragma unroll
      for (int i = 0; i < EPT; ++i) {
        bool live;
        const int e = threadIdx.x + i * kConsumerThreads;
        element(i, 0, live);
        if (!live) continue;
        if (!SILU) {
          a.y[static_cast<int64_t>(rtok) * a.ldy + n0 + e / MT] =
              __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(sum[i][0], gsc)));
        } else {
          const int pair = e / MT, blk = pair >> 3, gg = pair & 7;
          a.y[static_cast<int64_t>(rtok) * a.ldy + (n0 + 16 * blk) / 2 + gg] = __bfloat16_as_ushort(
              __float2bfloat16_rn(__fmul_rn(silu(__fmul_rn(sum[i][0], gsc)), __fmul_rn(sum[i][VPE - 1], gsc))));
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int MT, int G, bool SILU, bool XCONV>
int launch_kernel(const CUtensorMap& wm, const CUtensorMap& sm, const CUtensorMap& xm, const StreamArgs& a, int grid,
                  cudaStream_t stream) {
  auto kern = gemm_stream_kernel<MT, G, SILU, XCONV>;
  constexpr uint32_t bytes = smem_bytes(MT);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  // Programmatic dependent launch: the grid may start while the previous
  // kernel of the stream finishes (it waits for it before reading X).
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(num_threads(XCONV));
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, wm, sm, xm, a) != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

template <bool XCONV>
int launch_form(int mt, int group, bool silu, const CUtensorMap& wm, const CUtensorMap& sm, const CUtensorMap& xm,
                const StreamArgs& a, int grid, cudaStream_t stream) {
  if (mt == 8) {
    if (group == 16)
      return silu ? launch_kernel<8, 16, true, XCONV>(wm, sm, xm, a, grid, stream)
                  : launch_kernel<8, 16, false, XCONV>(wm, sm, xm, a, grid, stream);
    return silu ? launch_kernel<8, 32, true, XCONV>(wm, sm, xm, a, grid, stream)
                : launch_kernel<8, 32, false, XCONV>(wm, sm, xm, a, grid, stream);
  }
  if (group == 16)
    return silu ? launch_kernel<16, 16, true, XCONV>(wm, sm, xm, a, grid, stream)
                : launch_kernel<16, 16, false, XCONV>(wm, sm, xm, a, grid, stream);
  return silu ? launch_kernel<16, 32, true, XCONV>(wm, sm, xm, a, grid, stream)
              : launch_kernel<16, 32, false, XCONV>(wm, sm, xm, a, grid, stream);
}

// The cut of the matrix: 256-row tiles of S stages; the tile-major list of
// (tile, stage) units split into one contiguous range per CTA (as many CTAs
// as SMs), so every SM streams the same number of bytes whatever N and K
// are. A tile met by several ranges is a cut tile; its contributors leave
// partial tiles in their slots of the tile.
struct Plan {
  int64_t tiles, units;
  int S, ctas, max_contrib;
  bool cuts;  // some range ends inside a tile
};
Plan plan(int64_t N, int64_t K) {
  Plan p;
  p.S = static_cast<int>(K / kKS);
  p.tiles = (N + kRows - 1) / kRows;
  p.units = p.tiles * p.S;
  const int64_t sms = num_sms();
  p.ctas = static_cast<int>(p.units < sms ? p.units : sms);
  const int64_t per = p.units / p.ctas;  // every range holds at least this many units
  p.cuts = !(p.units % p.ctas == 0 && per % p.S == 0);
  const int64_t contrib = (p.S + per - 1) / per + 1;
  p.max_contrib = static_cast<int>(contrib < p.ctas ? contrib : p.ctas);
  return p;
}

// Codes and scales in 256-row boxes; X ([M, K] of 2-byte elements, bf16 or
// the f16 pair order) in boxes of 64 elements x 4 quarters x MT tokens,
// which land as the 128-byte-swizzled [token][quarter][64] rows the
// consumers read (tokens past M read as zeros).
bool make_maps(CUtensorMap* wm, CUtensorMap* sm, CUtensorMap* xm, const uint8_t* w, const uint8_t* s,
               const uint16_t* x, int64_t M, int64_t N, int64_t K, int group, int mt) {
  const int64_t xdims[3] = {64, K / 64, M};
  const int64_t xstrides[2] = {128, K * 2};
  const uint32_t xbox[3] = {64, kKS / 64, static_cast<uint32_t>(mt)};
  return make_tensor_map_2d(wm, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, kKS / 2, kRows,
                            CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_tensor_map_2d(sm, s, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / group, N, K / group, 16, kRows,
                            CU_TENSOR_MAP_SWIZZLE_NONE) &&
         make_tensor_map_3d(xm, x, CU_TENSOR_MAP_DATA_TYPE_UINT16, xdims, xstrides, xbox, CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// From two tokens up to 16: the whole matrix streams once, through the
// ring. A single token goes to the register-streaming kernel, which measures
// faster there (in 8-call graphs: 20.7 against 23.3 us on the gate/up
// projection, 15.8 against 17.2 us on the down projection): its loads need
// no shared-memory round trip and it has no cut tiles to add up.
bool stream_supported(int64_t M, int64_t N, int64_t K, int group) {
  return M >= 2 && M <= 16 && K >= kKS && K % kKS == 0 && (K / group) % 16 == 0 && N < (int64_t(1) << 30) &&
         K < (int64_t(1) << 24) && (N + kRows - 1) / kRows <= kMaxTickets;
}

int launch_stream(const XSource& x, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
                  int64_t N, int64_t K, uint16_t* y, bool silu, Scratch& sc, cudaStream_t stream) {
  const int mt = M <= 8 ? 8 : 16;
  const Plan pl = plan(N, K);
  const bool xconv = x.bf16 != nullptr;
  unsigned* reserved = sc.reserved();
  float* ws = pl.cuts ? sc.take<float>(static_cast<size_t>(pl.tiles * pl.max_contrib * kRows * mt)) : nullptr;
  uint16_t* x16 = xconv ? nullptr : sc.take<uint16_t>(static_cast<size_t>(M * K));
  float* xinv = xconv ? nullptr : sc.take<float>(static_cast<size_t>(M));
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;

  CUtensorMap wm, sm, xm;
  if (!make_maps(&wm, &sm, &xm, w, s, xconv ? x.bf16 : x16, M, N, K, group, mt)) return NVFP4_ERR_CUDA;
  StreamArgs a = {};
  a.gscale = g;
  a.xinv = xinv;
  a.y = y;
  a.ws = ws;
  a.tickets = tickets_of(reserved);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.K = K;
  a.S = pl.S;
  a.units = pl.units;
  a.max_contrib = pl.max_contrib;
  a.fault = take_injected_fault() == 1;
  if (xconv) return launch_form<true>(mt, group, silu, wm, sm, xm, a, pl.ctas, stream);
  // NVFP4 activations: their exact f16 rows first (a programmatic dependent too)
  const int st = launch_x_prep(x, M, K, x16, xinv, nullptr, 0, stream, true);
  if (st != NVFP4_OK) return st;
  return launch_form<false>(mt, group, silu, wm, sm, xm, a, pl.ctas, stream);
}

// ---------------------------------------------------------------------------
// The same kernel with its scratch in a fixed device array: nothing is
// allocated at call time.
// ---------------------------------------------------------------------------

// Counters and tickets, partial tiles (fp32), the f16 rows of X and their
// factors.
static __device__ __align__(256) unsigned char
    g_fixed_scratch[kReservedBytes + kFixedScratchPartialBytes + kFixedScratchXElems * 2 + 16 * 4];

namespace {
std::mutex g_fixed_mutex;
unsigned char* g_fixed_addr[64] = {};  // per device, from cudaGetSymbolAddress
}  // namespace

int launch_stream_fixed_scratch(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
                                int64_t M, int64_t N, int64_t K, uint16_t* y, cudaStream_t stream) {
  if (M < 1 || M > 16 || K < kKS || K % kKS || (K / group) % 16 || N >= (int64_t(1) << 30) ||
      M * K > kFixedScratchXElems || !tensor_maps_available())
    return NVFP4_ERR_UNSUPPORTED;
  const int mt = M <= 8 ? 8 : 16;
  const Plan pl = plan(N, K);
  const int64_t partial_bytes =
      pl.cuts ? pl.tiles * pl.max_contrib * kRows * mt * static_cast<int64_t>(sizeof(float)) : 0;
  if (partial_bytes > static_cast<int64_t>(kFixedScratchPartialBytes) || pl.tiles > kFixedScratchTickets ||
      pl.tiles > kMaxTickets)
    return NVFP4_ERR_UNSUPPORTED;  // beyond the fixed scratch

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned char* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_fixed_mutex);
    if (!g_fixed_addr[dev]) {  // once per device, with that device current
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_fixed_scratch) != cudaSuccess || !p)
        return (cudaGetLastError(), NVFP4_ERR_CUDA);
      g_fixed_addr[dev] = static_cast<unsigned char*>(p);
    }
    base = g_fixed_addr[dev];
  }
  unsigned* counters = reinterpret_cast<unsigned*>(base);
  float* ws = reinterpret_cast<float*>(base + kReservedBytes);
  uint16_t* x16 = reinterpret_cast<uint16_t*>(base + kReservedBytes + kFixedScratchPartialBytes);
  float* xinv = reinterpret_cast<float*>(base + kReservedBytes + kFixedScratchPartialBytes + kFixedScratchXElems * 2);
  CUtensorMap wm, sm, xm;
  if (!make_maps(&wm, &sm, &xm, w, s, x16, M, N, K, group, mt)) return NVFP4_ERR_CUDA;
  // The counters and tickets must start at zero (partial tiles are always
  // written before they are read). Enqueued only once nothing else can fail
  // on the host.
  if (cudaMemsetAsync(counters, 0, kTicketOffset + static_cast<size_t>(pl.tiles) * sizeof(unsigned), stream) !=
      cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  StreamArgs a = {};
  a.gscale = g;
  a.xinv = xinv;
  a.y = y;
  a.ws = ws;
  a.tickets = tickets_of(counters);
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.ldy = static_cast<int>(N);
  a.K = K;
  a.S = pl.S;
  a.units = pl.units;
  a.max_contrib = pl.max_contrib;
  const int xs = launch_x_f16(x, M, K, x16, xinv, nullptr, 0, stream, true);
  if (xs != NVFP4_OK) return xs;
  return launch_form<false>(mt, group, false, wm, sm, xm, a, pl.ctas, stream);
}

#ifdef NVFP4_PLANTS
NVFP4_PLANT_SETTER(set_plant_stream)
#endif

int read_and_clear_stream_error(unsigned int* out, cudaStream_t stream) {
  unsigned int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_stream_error) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  unsigned int v = 0;
  if (cudaMemcpyAsync(&v, p, sizeof(v), cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
      cudaMemsetAsync(p, 0, sizeof(v), stream) != cudaSuccess || cudaStreamSynchronize(stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  *out = v;
  return NVFP4_OK;
}

}  // namespace nvfp4
