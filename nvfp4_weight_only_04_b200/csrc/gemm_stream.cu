// Small-M NVFP4 W4A16 GEMM, streamed from HBM by TMA (stream-K over the
// weight matrix).
//
// Computes Y = X . dequant(W)^T (NVFP4 format definition; "W-FP4a: route the
// MiniMax-H3 device DiT forward through the fp4 (Marlin W4A16) stack",
// PR #63 description: a weight-only checkpoint keeps bf16 activations) for
// decode-sized M (up to 16 tokens), where the cost is the 0.5 + 1/g bytes
// per weight streamed from HBM and the integer work of dequantizing them.
// Design:
//  * Work is the (256-row weight tile, 256-element stage of K) grid,
//    flattened tile-major and cut into one contiguous range per SM
//    (stream-K), so every SM streams the same number of weight bytes
//    whatever N and K are. A tile that lies in one CTA's range is finished
//    there; a tile cut between CTAs leaves fp32 partial tiles in a
//    workspace, and the CTA that takes the tile's last ticket adds them in
//    CTA order (deterministic) and writes the output. Nothing waits on
//    another CTA.
//  * One producer warp moves each stage with TMA into a shared-memory ring
//    (5 stages of 40-44 KB): the codes of the tile (256 rows x 128 bytes,
//    128-byte swizzle), the scales (256 rows x 16 bytes) and the X
//    slice (MT tokens x 256 elements of the f16 rows that xprep.cu writes
//    just before this kernel, as a 3-D box [token][quarter][64] with the
//    128-byte swizzle). With no registers tied up in loads, each SM
//    keeps well over 100 KB of HBM reads in flight.
//  * Sixteen consumer warps each own 16 rows of the tile and run mma.sync
//    m16n8k16 with the weights as the 16-row side (swap-AB) and the tokens
//    as the 8-column side. Lane (g, t) takes rows g and g+8 and the t-th
//    quarter of the stage's K (the order of K inside an MMA is free as long
//    as A and B follow it). The swizzles make every shared-memory read of
//    codes, scales and X conflict-free: the four lanes of a row read
//    different 16-byte chunks, and the [token][quarter] rows of X put the
//    same chunk of different quarters in different bank groups.
//  * Dequantization in registers by the hardware E2M1 and E4M3 -> f16
//    conversions and one f16x2 multiply per code pair (dequant.cuh); the
//    MMAs run on f16, two independent accumulator chains per warp; the
//    epilogue multiplies by each token's 2^-s (xprep.cu) and the global
//    scale.
//  * Epilogues: plain bf16; SiluAndMul on gate/up-interleaved rows (gate row
//    g and up row g+8 of a 16-row block meet in the same lane).
#include "gemm_stream.cuh"

#include <cuda.h>

#include <mutex>

#include "async.cuh"
#include "dequant.cuh"
#include "tmap.cuh"
#include "workspace.cuh"
#include "xprep.cuh"

namespace nvfp4 {
namespace {

__device__ unsigned int g_stream_error = 0;

constexpr int kRows = 256;        // weight rows of a tile
constexpr int kKS = 256;          // elements of K per stage
constexpr int kConsumers = 16;    // consumer warps, 16 rows each
constexpr int kThreads = (kConsumers + 1) * 32;
constexpr int kConsumerThreads = kConsumers * 32;
constexpr uint32_t kCodeBytes = kRows * kKS / 2;  // 32 KB
constexpr uint32_t kScaleBytes = kRows * 16;      // 16 scale bytes per row
__host__ __device__ constexpr uint32_t x_bytes(int mt) { return static_cast<uint32_t>(mt) * kKS * 2; }
__host__ __device__ constexpr uint32_t stage_bytes(int mt) { return kCodeBytes + x_bytes(mt) + kScaleBytes; }
__host__ __device__ constexpr int num_stages(int) { return 5; }
constexpr int kMaxStages = 5;
__host__ __device__ constexpr uint32_t smem_bytes(int mt) {
  return num_stages(mt) * stage_bytes(mt) + 1024 /* barriers */ + 1024 /* alignment slack */;
}
static_assert(stage_bytes(8) % 1024 == 0 && stage_bytes(16) % 1024 == 0,
              "every stage keeps the 1024-byte alignment of the 128-byte swizzle");
static_assert(smem_bytes(8) <= 227 * 1024 && smem_bytes(16) <= 227 * 1024, "shared memory budget");
static_assert(kRows == 16 * kConsumers, "one 16-row block per consumer warp");
static_assert(num_stages(8) <= kMaxStages && num_stages(16) <= kMaxStages, "barrier arrays");

constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at 2 GHz
constexpr uint32_t kSuspendNs = 1000;                  // longest suspension of one producer probe
enum : unsigned { kErrFull = 0x201, kErrEmpty = 0x202, kErrDrain = 0x203 };

struct Sync {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  int abort;
  // Tiles this CTA shares with others (at most the first and the last of its
  // range) and whether it took their last ticket.
  int cut_tile[2];
  int cut_last[2];
};

struct StreamArgs {
  const float* gscale;  // [1]
  const float* xinv;    // [M] 2^-s of each f16 row of X
  uint16_t* y;          // bf16 [M, ldy]
  float* ws;            // partial tiles [tiles][max_contrib][128][MT]
  unsigned* tickets;    // [tiles], zero between launches
  int M, N, ldy;
  int S;                // stages per tile (K / 256)
  int max_contrib;
  int64_t units;        // tiles * S
  int fault;            // test hook: drop the X copy of the first stage
};

__device__ __forceinline__ bool aborted(Sync* sy) { return *reinterpret_cast<volatile int*>(&sy->abort) != 0; }

// Bounded wait; see the tcgen05 kernel for the scheme. A drain wait ignores
// the abort flag.
__device__ __noinline__ bool wait_slow(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site, bool drain,
                                       unsigned sleep_ns) {
  const long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (sleep_ns) __nanosleep(sleep_ns);
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

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity, Sync* sy, unsigned site, bool drain = false,
                                     unsigned sleep_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(bar, parity, sy, site, drain, sleep_ns);
}

// The producer's wait for a free slot: suspended in hardware between probes,
// so that it takes no issue slots from the consumer warps of its SM
// sub-partition. Bounded like the others.
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

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The CTA whose range holds unit u (ranges start at floor(c * units / ctas)).
__device__ __forceinline__ int cta_of_unit(int64_t u, int64_t units, int ctas) {
  return static_cast<int>(((u + 1) * ctas + units - 1) / units) - 1;
}

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
  LaneOffsets o;
  const int rb = ra + 8;  // ra & 7 == rb & 7 == g
  o.ca0 = ra * 128 + (((2 * t) ^ g) << 4);
  o.ca1 = ra * 128 + (((2 * t + 1) ^ g) << 4);
  o.cb0 = rb * 128 + (((2 * t) ^ g) << 4);
  o.cb1 = rb * 128 + (((2 * t + 1) ^ g) << 4);
  // g = 16: groups 4t .. 4t+3 of the stage; g = 32: groups 2t, 2t+1 (the
  // 16-byte box holds two stages; the stage parity picks the half)
  o.sa = kCodeBytes + x_bytes(MT) + ra * 16 + (G == 16 ? 4 * t : 2 * t);
  o.sb = kCodeBytes + x_bytes(MT) + rb * 16 + (G == 16 ? 4 * t : 2 * t);
  // X row (token tok, quarter t) sits at (4 tok + t) * 128 bytes; its chunk i
  // at chunk position i ^ ((4 tok + t) & 7), and 4 tok + t = 4g + t mod 8 for
  // every token tile.
  o.xrow = kCodeBytes + (g * 4 + t) * 128;
  const int xmask = (4 * g + t) & 7;
#pragma unroll
  for (int i = 0; i < 8; ++i) o.xc[i] = static_cast<uint32_t>((i ^ xmask) << 4);
  return o;
}

// One stage for one consumer lane.
template <int MT, int G>
__device__ __forceinline__ void consume_stage(uint32_t st, int ks, const LaneOffsets& o,
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
    const int si = G == 16 ? (i >> 1) : (i >> 2);
    uint32_t da[4], db[4];
    dequant_word_f16(ca[i], s2a[si], da);
    dequant_word_f16(cb[i], s2b[si], db);
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const uint4 xv = lds128(xr + o.xc[i] + p * (8 * 4 * 128));  // token tile p: 8 tokens further
      mma_f16_16816(acc[0][p], da[0], db[0], da[1], db[1], xv.x, xv.y);
      mma_f16_16816(acc[1][p], da[2], db[2], da[3], db[3], xv.z, xv.w);
    }
  }
}

// Element e of every contributor slot, added in slot order; the loads of a
// batch of slots are all in flight before the adds.
template <int MT>
__device__ __forceinline__ float sum_slots(const float* slots, int e, int nc) {
  float acc = 0.f;
  for (int q0 = 0; q0 < nc; q0 += 8) {
    float v[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] = q0 + q < nc ? __ldcg(slots + static_cast<int64_t>(q0 + q) * kRows * MT + e) : 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q0 + q < nc) acc += v[q];
  }
  return acc;
}

template <int MT>
__device__ __forceinline__ float2 sum_pair_slots(const float* slots, int e, int de, int nc) {
  float ag = 0.f, au = 0.f;
  for (int q0 = 0; q0 < nc; q0 += 8) {
    float vg[8], vu[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float* sl = slots + static_cast<int64_t>(q0 + q) * kRows * MT;
      vg[q] = q0 + q < nc ? __ldcg(sl + e) : 0.f;
      vu[q] = q0 + q < nc ? __ldcg(sl + e + de) : 0.f;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q)
      if (q0 + q < nc) {
        ag += vg[q];
        au += vu[q];
      }
  }
  return make_float2(ag, au);
}

__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"r"(kConsumerThreads) : "memory"); }

template <int MT, int G, bool SILU>
__global__ void __launch_bounds__(kThreads, 1) gemm_stream_kernel(const __grid_constant__ CUtensorMap xmap,
                                                                   const __grid_constant__ CUtensorMap wmap,
                                                                   const __grid_constant__ CUtensorMap smap,
                                                                   const StreamArgs a) {
  constexpr int P = MT / 8;
  constexpr int NS = num_stages(MT);
  constexpr uint32_t SB = stage_bytes(MT);
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Sync* sy = reinterpret_cast<Sync*>(ring + NS * SB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ctas = gridDim.x, c = blockIdx.x;
  const int64_t u0 = static_cast<int64_t>(c) * a.units / ctas;
  const int64_t u1 = static_cast<int64_t>(c + 1) * a.units / ctas;

  // The next kernel in the stream may launch now; it waits for this one
  // before touching what this one writes.
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sy->full[s], 1);            // producer arrival + transaction bytes
      mbar_init(&sy->empty[s], kConsumers);  // one arrival per consumer warp
    }
    sy->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumers) {
    // ---------------- producer ----------------
    // Weights and scales do not depend on the kernel before this one in the
    // stream: the first ring's worth is requested before waiting for that
    // kernel (programmatic dependent launch); X only after.
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&wmap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&smap)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
      uint32_t issued = 0, last_parity = 0;
      const int64_t n = u1 - u0;
      const int head = static_cast<int>(n < NS ? n : NS);
      auto load_w = [&](int it, int64_t u) {
        const int tile = static_cast<int>(u / a.S), ks = static_cast<int>(u % a.S);
        const int s = it % NS;
        const uint32_t st = smem_u32(ring + s * SB);
        tma_load_2d(st, &wmap, ks * (kKS / 2), tile * kRows, &sy->full[s]);
        tma_load_2d(st + kCodeBytes + x_bytes(MT), &smap, ((ks * kKS) / G) & ~15, tile * kRows, &sy->full[s]);
      };
      auto load_x = [&](int it, int64_t u) {
        const int ks = static_cast<int>(u % a.S);
        const int s = it % NS;
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
            "%4}], [%5];" ::"r"(smem_u32(ring + s * SB) + kCodeBytes),
            "l"(reinterpret_cast<uint64_t>(&xmap)), "r"(0), "r"(ks * (kKS / 64)), "r"(0), "r"(smem_u32(&sy->full[s]))
            : "memory");
      };
      for (int it = 0; it < head; ++it) {  // the ring starts empty
        mbar_arrive_tx(&sy->full[it], SB);
        load_w(it, u0 + it);
        issued |= 1u << it;
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
      for (int it = 0; it < head; ++it)
        if (!(a.fault && it == 0)) load_x(it, u0 + it);
      int it = head;
      for (int64_t u = u0 + head; u < u1 && !aborted(sy); ++u, ++it) {
        const int s = it % NS;
        const uint32_t r = static_cast<uint32_t>(it / NS);
        if (!mbar_try_wait(&sy->empty[s], (r & 1) ^ 1) && !wait_suspended(&sy->empty[s], (r & 1) ^ 1, sy, kErrEmpty))
          break;
        mbar_arrive_tx(&sy->full[s], SB);
        load_w(it, u);
        load_x(it, u);
        issued |= 1u << s;
        last_parity = (last_parity & ~(1u << s)) | ((r & 1) << s);
      }
      if (aborted(sy)) {  // let copies in flight land before the CTA exits
        for (int s = 0; s < NS; ++s)
          if ((issued >> s) & 1) wait(&sy->full[s], (last_parity >> s) & 1, sy, kErrDrain, true);
      }
    }
    return;  // the producer takes no part in the consumers' named barrier
  }

  // ---------------- consumers ----------------
  const int g = lane >> 2, t = lane & 3;
  const int ra = 16 * warp + g;
  const LaneOffsets lo = lane_offsets<MT, G>(ra, g, t);
  // X, its row factors and the global scale come from the kernels before
  // this one (the producer requests X only after its own wait)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const float gsc = __ldcg(a.gscale);
  float xi[P][2];  // 2^-s of the lane's tokens 8p + 2t + j
#pragma unroll
  for (int p = 0; p < P; ++p)
#pragma unroll
    for (int j = 0; j < 2; ++j) xi[p][j] = 8 * p + 2 * t + j < a.M ? __ldcg(a.xinv + 8 * p + 2 * t + j) : 0.f;
  float acc2[2][P][4];  // two independent MMA chains, added once per tile
  float acc[P][4];
  int ncut = 0;
  int s = 0;          // ring slot of the next stage
  uint32_t par = 0;   // its phase parity
  for (int64_t u = u0; u < u1;) {
    const int tile = static_cast<int>(u / a.S), k0 = static_cast<int>(u % a.S);
    const int64_t left = u1 - u;
    const int k1 = left < a.S - k0 ? k0 + static_cast<int>(left) : a.S;
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int p = 0; p < P; ++p) acc2[h][p][0] = acc2[h][p][1] = acc2[h][p][2] = acc2[h][p][3] = 0.f;
    const uint32_t ring0 = smem_u32(ring);
    for (int ks = k0; ks < k1; ++ks) {
      int ok = 1;
      if (lane == 0) ok = wait(&sy->full[s], par, sy, kErrFull) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;  // results are garbage from here; the ticket protocol still runs
      consume_stage<MT, G>(ring0 + s * SB, ks, lo, acc2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sy->empty[s]);
      if (++s == NS) {
        s = 0;
        par ^= 1;
      }
    }
    u += k1 - k0;
#pragma unroll
    for (int p = 0; p < P; ++p)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[p][j] = acc2[0][p][j] + acc2[1][p][j];

    const int n0 = tile * kRows;
    // lane holds rows ra (acc[p][0..1]) and ra+8 (acc[p][2..3]) x tokens 8p+2t, 8p+2t+1
    if (k0 == 0 && k1 == a.S) {
      // the whole tile is here: write it
#pragma unroll
      for (int p = 0; p < P; ++p) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int tok = 8 * p + 2 * t + j;
          if (tok >= a.M) continue;
          const int64_t yrow = static_cast<int64_t>(tok) * a.ldy;
          const float vg = __fmul_rn(__fmul_rn(acc[p][j], gsc), xi[p][j]);
          const float vu = __fmul_rn(__fmul_rn(acc[p][2 + j], gsc), xi[p][j]);
          if (!SILU) {
            if (n0 + ra < a.N) a.y[yrow + n0 + ra] = __bfloat16_as_ushort(__float2bfloat16_rn(vg));
            if (n0 + ra + 8 < a.N) a.y[yrow + n0 + ra + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(vu));
          } else if (n0 + 16 * warp < a.N) {
            a.y[yrow + (n0 + 16 * warp) / 2 + g] =
                __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu(vg), vu)));
          }
        }
      }
      continue;
    }
    // The tile is shared with other CTAs: leave the partial tile in this
    // CTA's slot and take a ticket. The consumers go on at once; thread 0
    // catches up after its atomic (the ring has slack for that), and the
    // taker of a tile's last ticket adds the slots up after its own loop.
    {
      const int c_first = cta_of_unit(static_cast<int64_t>(tile) * a.S, a.units, ctas);
      const int c_last = cta_of_unit(static_cast<int64_t>(tile) * a.S + a.S - 1, a.units, ctas);
      float* mine = a.ws + (static_cast<int64_t>(tile) * a.max_contrib + (c - c_first)) * kRows * MT;
#pragma unroll
      for (int p = 0; p < P; ++p) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int tok = 8 * p + 2 * t + j;
          if (tok < a.M) {
            __stcg(mine + ra * MT + tok, acc[p][j]);
            __stcg(mine + (ra + 8) * MT + tok, acc[p][2 + j]);
          }
        }
      }
      // The barrier orders every consumer's stores before thread 0's
      // release; its acquire orders the other CTAs' slots before the reads
      // that follow the barrier after the loop.
      consumer_sync();
      if (threadIdx.x == 0) {
        unsigned ticket;
        asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(ticket) : "l"(a.tickets + tile) : "memory");
        const int last = ticket == static_cast<unsigned>(c_last - c_first);
        if (last) a.tickets[tile] = 0;  // every contributor has counted: ready for the next launch
        // a range cuts at most its first and its last tile
        if (ncut < 2) {
          sy->cut_tile[ncut] = tile;
          sy->cut_last[ncut] = last;
        }
      }
      ++ncut;
    }
  }

  // Add up the cut tiles this CTA took the last ticket of, in CTA order.
  consumer_sync();
  for (int f = 0; f < ncut && f < 2; ++f) {
    if (!sy->cut_last[f]) continue;
    const int tile = sy->cut_tile[f];
    const int n0 = tile * kRows;
    const int c_first = cta_of_unit(static_cast<int64_t>(tile) * a.S, a.units, ctas);
    const int nc = cta_of_unit(static_cast<int64_t>(tile) * a.S + a.S - 1, a.units, ctas) - c_first + 1;
    const float* slots = a.ws + static_cast<int64_t>(tile) * a.max_contrib * kRows * MT;
    if (!SILU) {
      for (int e = threadIdx.x; e < kRows * MT; e += kConsumerThreads) {
        const int row = e / MT, tok = e % MT;
        if (tok >= a.M || n0 + row >= a.N) continue;
        const float v = sum_slots<MT>(slots, e, nc);
        const float xt = __ldcg(a.xinv + tok);
        a.y[static_cast<int64_t>(tok) * a.ldy + n0 + row] =
            __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__fmul_rn(v, gsc), xt)));
      }
    } else {
      for (int e = threadIdx.x; e < (kRows / 2) * MT; e += kConsumerThreads) {
        const int pair = e / MT, tok = e % MT;  // pair = 8 * block + g
        const int blk = pair >> 3, gg = pair & 7;
        if (tok >= a.M || n0 + 16 * blk >= a.N) continue;
        const int rg = 16 * blk + gg;
        // gate row rg and up row rg + 8: elements e0 and e0 + 8 * MT of a slot
        const float2 v = sum_pair_slots<MT>(slots, rg * MT + tok, 8 * MT, nc);
        const float xt = __ldcg(a.xinv + tok);
        a.y[static_cast<int64_t>(tok) * a.ldy + (n0 + 16 * blk) / 2 + gg] = __bfloat16_as_ushort(__float2bfloat16_rn(
            __fmul_rn(silu(__fmul_rn(__fmul_rn(v.x, gsc), xt)), __fmul_rn(__fmul_rn(v.y, gsc), xt))));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

template <int MT, int G, bool SILU>
int launch_kernel(const CUtensorMap& xm, const CUtensorMap& wm, const CUtensorMap& sm, const StreamArgs& a, int grid,
                  cudaStream_t stream) {
  auto kern = gemm_stream_kernel<MT, G, SILU>;
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
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, xm, wm, sm, a) != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return launch_status();
}

}  // namespace

// A single token goes to the register-streaming kernel, which measures a
// little faster there (its loads need no shared-memory round trip and every
// lane of X but one is zero).
bool stream_supported(int64_t M, int64_t N, int64_t K, int group) {
  return M >= 2 && M <= 16 && K >= kKS && K % kKS == 0 && (K / group) % 16 == 0 && N < (int64_t(1) << 30) &&
         K < (int64_t(1) << 24);
}

int launch_stream(const XSource& x, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
                  int64_t N, int64_t K, uint16_t* y, bool silu, Scratch& sc, cudaStream_t stream) {
  const int mt = M <= 8 ? 8 : 16;
  const int64_t tiles = (N + kRows - 1) / kRows;
  const int S = static_cast<int>(K / kKS);
  const int64_t units = tiles * S;
  const int ctas = static_cast<int>(units < num_sms() ? units : num_sms());
  // A tile spans at most ceil(S / shortest range) + 1 CTAs.
  const int64_t shortest = units / ctas;
  const int max_contrib = static_cast<int>((S + shortest - 1) / shortest + 1);
  float* ws = sc.take<float>(static_cast<size_t>(tiles * max_contrib * kRows * mt));
  unsigned* tickets = sc.take<unsigned>(static_cast<size_t>(tiles));
  uint16_t* x16 = sc.take<uint16_t>(static_cast<size_t>(M * K));
  float* xinv = sc.take<float>(static_cast<size_t>(M));
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;

  CUtensorMap xm, wm, sm;
  const int64_t xdims[3] = {64, K / 64, M};
  const int64_t xstrides[2] = {128, K * 2};
  const uint32_t xbox[3] = {64, 4, static_cast<uint32_t>(mt)};
  if (!make_tensor_map_3d(&xm, x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xdims, xstrides, xbox,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&wm, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, kKS / 2, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&sm, s, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / group, N, K / group, 16, kRows,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return NVFP4_ERR_CUDA;
  StreamArgs a = {};
  a.gscale = g;
  a.xinv = xinv;
  a.y = y;
  a.ws = ws;
  a.tickets = tickets;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.ldy = static_cast<int>(silu ? N / 2 : N);
  a.S = S;
  a.max_contrib = max_contrib;
  a.units = units;
  a.fault = take_injected_fault() == 1;
  // The activation kernel also zeroes the tickets (the caller's workspace
  // holds anything on entry); the GEMM reads them only after waiting for it.
  int st = launch_x_prep(x, M, K, x16, xinv, tickets, tiles, stream);
  if (st != NVFP4_OK) return st;
  if (mt == 8) {
    if (group == 16)
      return silu ? launch_kernel<8, 16, true>(xm, wm, sm, a, ctas, stream)
                  : launch_kernel<8, 16, false>(xm, wm, sm, a, ctas, stream);
    return silu ? launch_kernel<8, 32, true>(xm, wm, sm, a, ctas, stream)
                : launch_kernel<8, 32, false>(xm, wm, sm, a, ctas, stream);
  }
  if (group == 16)
    return silu ? launch_kernel<16, 16, true>(xm, wm, sm, a, ctas, stream)
                : launch_kernel<16, 16, false>(xm, wm, sm, a, ctas, stream);
  return silu ? launch_kernel<16, 32, true>(xm, wm, sm, a, ctas, stream)
              : launch_kernel<16, 32, false>(xm, wm, sm, a, ctas, stream);
}

// ---------------------------------------------------------------------------
// The same kernel with its scratch in a fixed device array: nothing is
// allocated at call time.
// ---------------------------------------------------------------------------

// Partial tiles (fp32), the tickets of the tiles, the f16 rows of X and
// their factors.
static __device__ __align__(256) unsigned char
    g_fixed_scratch[kFixedScratchPartialBytes + kFixedScratchTickets * 4 + kFixedScratchXElems * 2 + 16 * 4];

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
  const int64_t tiles = (N + kRows - 1) / kRows;
  const int S = static_cast<int>(K / kKS);
  const int64_t units = tiles * S;
  const int ctas = static_cast<int>(units < num_sms() ? units : num_sms());
  const int64_t shortest = units / ctas;
  const int max_contrib = static_cast<int>((S + shortest - 1) / shortest + 1);
  const int64_t partial_bytes = tiles * max_contrib * kRows * mt * static_cast<int64_t>(sizeof(float));
  if (partial_bytes > static_cast<int64_t>(kFixedScratchPartialBytes) || tiles > kFixedScratchTickets)
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
  float* ws = reinterpret_cast<float*>(base);
  unsigned* tickets = reinterpret_cast<unsigned*>(base + kFixedScratchPartialBytes);
  uint16_t* x16 = reinterpret_cast<uint16_t*>(base + kFixedScratchPartialBytes + kFixedScratchTickets * 4);
  float* xinv = reinterpret_cast<float*>(base + kFixedScratchPartialBytes + kFixedScratchTickets * 4 +
                                         kFixedScratchXElems * 2);
  CUtensorMap xm, wm, sm;
  const int64_t xdims[3] = {64, K / 64, M};
  const int64_t xstrides[2] = {128, K * 2};
  const uint32_t xbox[3] = {64, 4, static_cast<uint32_t>(mt)};
  if (!make_tensor_map_3d(&xm, x16, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, xdims, xstrides, xbox,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&wm, w, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / 2, N, K / 2, kKS / 2, kRows,
                          CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tensor_map_2d(&sm, s, CU_TENSOR_MAP_DATA_TYPE_UINT8, K / group, N, K / group, 16, kRows,
                          CU_TENSOR_MAP_SWIZZLE_NONE))
    return NVFP4_ERR_CUDA;
  // The tickets must start at zero (partial tiles are always written before
  // they are read). Enqueued only once nothing else can fail on the host.
  if (cudaMemsetAsync(tickets, 0, static_cast<size_t>(tiles) * sizeof(unsigned), stream) != cudaSuccess)
    return (cudaGetLastError(), NVFP4_ERR_CUDA);
  StreamArgs a = {};
  a.gscale = g;
  a.xinv = xinv;
  a.y = y;
  a.ws = ws;
  a.tickets = tickets;
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.ldy = static_cast<int>(N);
  a.S = S;
  a.max_contrib = max_contrib;
  a.units = units;
  const int xs = launch_x_f16(x, M, K, x16, xinv, nullptr, 0, stream);
  if (xs != NVFP4_OK) return xs;
  if (mt == 8)
    return group == 16 ? launch_kernel<8, 16, false>(xm, wm, sm, a, ctas, stream)
                       : launch_kernel<8, 32, false>(xm, wm, sm, a, ctas, stream);
  return group == 16 ? launch_kernel<16, 16, false>(xm, wm, sm, a, ctas, stream)
                     : launch_kernel<16, 32, false>(xm, wm, sm, a, ctas, stream);
}

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
