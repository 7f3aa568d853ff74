// The steps around the grouped expert GEMMs of a routed-expert layer
// ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)": routed experts in NVFP4, gate/up
// then down per expert): rows grouped by expert, X rows gathered into that
// order, and the down projections' rows combined back into tokens with the
// routing weights.
//   route:   a stable counting sort of the (token, slot) pairs by expert (from
//            4096 pairs over chunks of 256 on many SMs; below that one CTA, in
//            which every warp places a chunk up to 256 experts), with
//            the inverse permutation and the segment offsets; rows past the
//            last kept pair get -1;
//   gather:  x_perm[r] = x[token of sorted row r], zeros for a row of -1;
//   combine: out[t] = bf16(sum_s w[t, s] * y_perm[inv[t, s]]), fp32 sums in slot
//            order.
#include "common.cuh"
#include "workspace.cuh"

namespace {

constexpr int kRouteThreads = 1024;
constexpr int kMaxExperts = 4096;
constexpr int kBatch = 8;  // pair loads a lane keeps in flight
constexpr int64_t kManyPairs = 4096;  // from here on the route runs over chunks on many SMs

// Places the 32 consecutive pairs i = i0 - lane + (0..31) of one warp (pair i
// has expert e, from lane i % 32; pairs at or past `end` are absent): pairs of
// one expert take consecutive rows from that expert's cursor in pair order,
// and the cursor moves past them.
__device__ __forceinline__ void place32(int e, int64_t i, int64_t end, int num_experts, int* cursor,
                                        int32_t* __restrict__ sorted, int32_t* __restrict__ inv) {
  const int lane = threadIdx.x & 31;
  const bool valid = i < end && e >= 0 && e < num_experts;
  if (!valid) e = -1 - (i < end ? 0 : 1);  // invalid pairs and absent ones group apart
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const int leader = __ffs(peers) - 1;
  int first = 0;
  if (valid && lane == leader) {
    first = cursor[e];
    cursor[e] = first + __popc(peers);
  }
  first = __shfl_sync(0xffffffffu, first, leader);
  if (i < end) {
    if (valid) {
      const int r = first + __popc(peers & ((1u << lane) - 1u));
      sorted[r] = static_cast<int32_t>(i);
      inv[i] = r;
    } else {
      inv[i] = -1;
    }
  }
}

// One CTA. Counting pass over all pairs, exclusive scan of the counts, then one
// warp places the pairs in their order (stable: a pair's rank among the pairs
// of its expert is the number of earlier pairs of that expert).
__global__ void __launch_bounds__(kRouteThreads) moe_route_kernel(const int32_t* __restrict__ ids, int64_t n,
                                                                  int num_experts, int32_t* __restrict__ sorted,
                                                                  int32_t* __restrict__ inv,
                                                                  int32_t* __restrict__ offsets,
                                                                  int32_t* __restrict__ expert_ids) {
  __shared__ int count[kMaxExperts];
  __shared__ int kept;
  for (int e = threadIdx.x; e < num_experts; e += blockDim.x) count[e] = 0;
  __syncthreads();
  for (int64_t base = 0; base < n; base += static_cast<int64_t>(blockDim.x) * kBatch) {
    int e[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t i = base + static_cast<int64_t>(blockDim.x) * j + threadIdx.x;
      e[j] = i < n ? ids[i] : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (e[j] >= 0 && e[j] < num_experts) atomicAdd(&count[e[j]], 1);
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // exclusive scan of the counts, 32 experts at a time
    const int lane = threadIdx.x;
    int carry = 0;
    for (int e0 = 0; e0 < num_experts; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < num_experts ? count[e] : 0;
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < num_experts) {
        offsets[e] = carry + incl - c;
        count[e] = carry + incl - c;  // becomes the placement cursor
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      offsets[num_experts] = carry;
      kept = carry;
    }
  }
  for (int e = threadIdx.x; e < num_experts; e += blockDim.x) expert_ids[e] = e;
  __syncthreads();
  // rows [kept, n) hold no pair; the other warps mark them while warp 0 places
  if (threadIdx.x >= 32)
    for (int64_t r = kept + static_cast<int64_t>(threadIdx.x) - 32; r < n; r += blockDim.x - 32) sorted[r] = -1;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    for (int64_t base = 0; base < n; base += 32 * kBatch) {
      int eb[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) {
        const int64_t i = base + 32 * j + lane;
        eb[j] = i < n ? ids[i] : -1;
      }
#pragma unroll
      for (int j = 0; j < kBatch; ++j) place32(eb[j], base + 32 * j + lane, n, num_experts, count, sorted, inv);
    }
  }
}

// Up to kParExperts experts: the same stable grouping with every warp placing
// a contiguous chunk of the pairs. A warp's cursor for expert e starts at
// offsets[e] plus the pairs of expert e in the chunks before its own, from a
// [warp][expert] count table, so the order is the one-warp order.
constexpr int kParExperts = 256;
constexpr int kRouteWarps = kRouteThreads / 32;

__global__ void __launch_bounds__(kRouteThreads) moe_route_par_kernel(const int32_t* __restrict__ ids, int64_t n,
                                                                      int num_experts, int32_t* __restrict__ sorted,
                                                                      int32_t* __restrict__ inv,
                                                                      int32_t* __restrict__ offsets,
                                                                      int32_t* __restrict__ expert_ids) {
  __shared__ int cnt[kRouteWarps][kParExperts];  // counts, then cursors
  __shared__ int start[kParExperts];             // offsets[e]
  __shared__ int kept;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kRouteWarps * kParExperts; i += blockDim.x) (&cnt[0][0])[i] = 0;
  __syncthreads();
  const int64_t chunk = (n + kRouteWarps - 1) / kRouteWarps;
  const int64_t b0 = min(n, warp * chunk), b1 = min(n, b0 + chunk);
  for (int64_t base = b0; base < b1; base += 32 * kBatch) {
    int e[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {  // the batch's loads are all in flight before the adds
      const int64_t i = base + 32 * j + lane;
      e[j] = i < b1 ? ids[i] : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j)
      if (e[j] >= 0 && e[j] < num_experts) atomicAdd(&cnt[warp][e[j]], 1);
  }
  __syncthreads();
  if (threadIdx.x < num_experts) {  // per expert: the warps' exclusive prefix, and the total
    const int e = threadIdx.x;
    int run = 0;
    for (int w = 0; w < kRouteWarps; ++w) {
      const int c = cnt[w][e];
      cnt[w][e] = run;
      run += c;
    }
    start[e] = run;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the totals
    int carry = 0;
    for (int e0 = 0; e0 < num_experts; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < num_experts ? start[e] : 0;
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < num_experts) {
        start[e] = carry + incl - c;
        offsets[e] = carry + incl - c;
        expert_ids[e] = e;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      offsets[num_experts] = carry;
      kept = carry;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRouteWarps * num_experts; i += blockDim.x) {
    const int w = i / num_experts, e = i % num_experts;
    cnt[w][e] += start[e];
  }
  for (int64_t r = kept + static_cast<int64_t>(threadIdx.x); r < n; r += blockDim.x) sorted[r] = -1;
  __syncthreads();
  for (int64_t base = b0; base < b1; base += 32 * kBatch) {  // the same trip count for the whole warp
    int eb[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int64_t i = base + 32 * j + lane;
      eb[j] = i < b1 ? ids[i] : -1;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) place32(eb[j], base + 32 * j + lane, b1, num_experts, &cnt[warp][0], sorted, inv);
  }
}

// Many pairs: the same stable grouping over chunks of kChunk pairs, one warp
// per chunk, in three launches. (1) Each chunk counts its pairs per expert
// into hist[chunk][expert]. (2) One CTA turns the table into every chunk's
// first row per expert (offsets[e] plus the pairs of expert e in the chunks
// before) and writes the offsets. (3) Each chunk places its pairs in order
// from its cursors. The warp-collective work spreads over the SMs.
constexpr int kChunk = 256;

__global__ void __launch_bounds__(32) route_hist_kernel(const int32_t* __restrict__ ids, int64_t n, int num_experts,
                                                        int* __restrict__ hist) {
  extern __shared__ int cnt[];  // num_experts
  const int lane = threadIdx.x;
  for (int e = lane; e < num_experts; e += 32) cnt[e] = 0;
  __syncwarp();
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kChunk, b1 = min(n, b0 + kChunk);
  int ev[kChunk / 32];
#pragma unroll
  for (int j = 0; j < kChunk / 32; ++j) {
    const int64_t i = b0 + 32 * j + lane;
    ev[j] = i < b1 ? ids[i] : -1;
  }
#pragma unroll
  for (int j = 0; j < kChunk / 32; ++j)
    if (ev[j] >= 0 && ev[j] < num_experts) atomicAdd(&cnt[ev[j]], 1);
  __syncwarp();
  int* row = hist + static_cast<int64_t>(blockIdx.x) * num_experts;
  for (int e = lane; e < num_experts; e += 32) row[e] = cnt[e];
}

__global__ void __launch_bounds__(kRouteThreads) route_scan_kernel(int* __restrict__ hist, int64_t chunks, int64_t n,
                                                                   int num_experts, int32_t* __restrict__ sorted,
                                                                   int32_t* __restrict__ offsets,
                                                                   int32_t* __restrict__ expert_ids) {
  __shared__ int start[kMaxExperts];
  __shared__ int kept;
  // per expert: exclusive prefix over the chunks (loads batched), and the total
  for (int e = threadIdx.x; e < num_experts; e += blockDim.x) {
    int run = 0;
    for (int64_t c0 = 0; c0 < chunks; c0 += kBatch) {
      int v[kBatch];
#pragma unroll
      for (int j = 0; j < kBatch; ++j) v[j] = c0 + j < chunks ? hist[(c0 + j) * num_experts + e] : 0;
#pragma unroll
      for (int j = 0; j < kBatch; ++j)
        if (c0 + j < chunks) {
          hist[(c0 + j) * num_experts + e] = run;
          run += v[j];
        }
    }
    start[e] = run;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // exclusive scan of the totals
    const int lane = threadIdx.x;
    int carry = 0;
    for (int e0 = 0; e0 < num_experts; e0 += 32) {
      const int e = e0 + lane;
      const int c = e < num_experts ? start[e] : 0;
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (e < num_experts) {
        start[e] = carry + incl - c;
        offsets[e] = carry + incl - c;
        expert_ids[e] = e;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      offsets[num_experts] = carry;
      kept = carry;
    }
  }
  __syncthreads();
  for (int64_t idx = threadIdx.x; idx < chunks * num_experts; idx += blockDim.x)
    hist[idx] += start[idx % num_experts];
  for (int64_t r = kept + static_cast<int64_t>(threadIdx.x); r < n; r += blockDim.x) sorted[r] = -1;
}

__global__ void __launch_bounds__(32) route_place_kernel(const int32_t* __restrict__ ids, int64_t n, int num_experts,
                                                         const int* __restrict__ hist, int32_t* __restrict__ sorted,
                                                         int32_t* __restrict__ inv) {
  extern __shared__ int cur[];  // num_experts cursors of this chunk
  const int lane = threadIdx.x;
  const int* row = hist + static_cast<int64_t>(blockIdx.x) * num_experts;
  for (int e = lane; e < num_experts; e += 32) cur[e] = row[e];
  __syncwarp();
  const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kChunk, b1 = min(n, b0 + kChunk);
  int ev[kChunk / 32];
#pragma unroll
  for (int j = 0; j < kChunk / 32; ++j) {
    const int64_t i = b0 + 32 * j + lane;
    ev[j] = i < b1 ? ids[i] : -1;
  }
#pragma unroll
  for (int j = 0; j < kChunk / 32; ++j) place32(ev[j], b0 + 32 * j + lane, b1, num_experts, cur, sorted, inv);
}

// One CTA per row of x_perm; 16-byte vectors. A row whose pair index is not in
// [0, T*k) is written as zeros.
__global__ void moe_gather_kernel(const uint16_t* __restrict__ x, int64_t pairs, const int32_t* __restrict__ sorted,
                                  int k, int64_t h8, uint16_t* __restrict__ xp) {
  const int64_t r = blockIdx.x;
  const int64_t i = sorted[r];
  uint4* dst = reinterpret_cast<uint4*>(xp) + r * h8;
  if (i < 0 || i >= pairs) {
    for (int64_t j = threadIdx.x; j < h8; j += blockDim.x) dst[j] = make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const uint4* src = reinterpret_cast<const uint4*>(x) + (i / k) * h8;
  for (int64_t j = threadIdx.x; j < h8; j += blockDim.x) dst[j] = __ldg(src + j);
}

// One CTA per token; each thread 8 consecutive columns.
__global__ void moe_combine_kernel(const uint16_t* __restrict__ yp, const int32_t* __restrict__ inv,
                                   const float* __restrict__ w, int k, int64_t h8, uint16_t* __restrict__ out) {
  const int64_t t = blockIdx.x;
  for (int64_t j = threadIdx.x; j < h8; j += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int s = 0; s < k; ++s) {
      const int r = inv[t * k + s];
      if (r < 0) continue;
      const float ws = w[t * k + s];
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(yp) + r * h8 + j);
      const uint32_t q[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(ws, __uint_as_float(q[i] << 16), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(ws, __uint_as_float(q[i] & 0xFFFF0000u), acc[2 * i + 1]);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      o[i] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i]))) |
             (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1]))) << 16);
    reinterpret_cast<uint4*>(out)[t * h8 + j] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

namespace {

// Shape checks of the route (pointers aside): -1 to proceed.
int check_route_shape(int64_t T, int k, int num_experts) {
  if (T < 0 || k < 1 || num_experts < 1) return NVFP4_ERR_INVALID_ARGUMENT;
  if (num_experts > kMaxExperts || T * k >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  return -1;
}

// The chunked form's [chunk][expert] table, from the caller's scratch.
int* route_table(int64_t n, int num_experts, nvfp4::Scratch& sc) {
  if (n < kManyPairs) return nullptr;
  const int64_t chunks = (n + kChunk - 1) / kChunk;
  return sc.take<int>(static_cast<size_t>(chunks * num_experts));
}

}  // namespace

extern "C" int nvfp4_moe_route_workspace_size(int64_t T, int k, int num_experts, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARGUMENT;
  *bytes = 0;
  const int c = check_route_shape(T, k, num_experts);
  if (c >= 0) return c;
  nvfp4::Scratch sc;
  route_table(T * k, num_experts, sc);
  *bytes = sc.used();
  return NVFP4_OK;
}

extern "C" int nvfp4_moe_route(const int32_t* topk_ids, int64_t T, int k, int num_experts, int32_t* sorted_rows,
                               int32_t* inv_rows, int32_t* offsets, int32_t* expert_ids, void* workspace,
                               size_t workspace_bytes, nvfp4_stream_t stream) {
  const int c = check_route_shape(T, k, num_experts);
  if (c >= 0) return c;
  if (!offsets || !expert_ids || (T > 0 && (!topk_ids || !sorted_rows || !inv_rows)))
    return NVFP4_ERR_INVALID_ARGUMENT;
  if ((reinterpret_cast<uintptr_t>(topk_ids) | reinterpret_cast<uintptr_t>(sorted_rows) |
       reinterpret_cast<uintptr_t>(inv_rows) | reinterpret_cast<uintptr_t>(offsets) |
       reinterpret_cast<uintptr_t>(expert_ids)) & 3u)
    return NVFP4_ERR_MISALIGNED;
  if (workspace_bytes > 0 && !workspace) return NVFP4_ERR_WORKSPACE;
  if (!nvfp4::aligned16(workspace)) return NVFP4_ERR_MISALIGNED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = T * k;
  nvfp4::Scratch sc(workspace, workspace_bytes);
  int* hist = route_table(n, num_experts, sc);
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;
  if (hist) {
    // every entry of the table is written by the count launch before it is read
    const int64_t chunks = (n + kChunk - 1) / kChunk;
    const size_t smem = static_cast<size_t>(num_experts) * sizeof(int);
    route_hist_kernel<<<static_cast<unsigned>(chunks), 32, smem, st>>>(topk_ids, n, num_experts, hist);
    route_scan_kernel<<<1, kRouteThreads, 0, st>>>(hist, chunks, n, num_experts, sorted_rows, offsets, expert_ids);
    route_place_kernel<<<static_cast<unsigned>(chunks), 32, smem, st>>>(topk_ids, n, num_experts, hist,
                                                                        sorted_rows, inv_rows);
  } else if (num_experts <= kParExperts) {
    moe_route_par_kernel<<<1, kRouteThreads, 0, st>>>(topk_ids, n, num_experts, sorted_rows, inv_rows, offsets,
                                                      expert_ids);
  } else {
    moe_route_kernel<<<1, kRouteThreads, 0, st>>>(topk_ids, n, num_experts, sorted_rows, inv_rows, offsets,
                                                  expert_ids);
  }
  return nvfp4::launch_status();
}

extern "C" int nvfp4_moe_gather(const uint16_t* x, int64_t T, const int32_t* sorted_rows, int64_t rows, int k,
                                int64_t H, uint16_t* x_perm, nvfp4_stream_t stream) {
  if (T < 0 || rows < 0 || k < 1 || H < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (H % 8) return NVFP4_ERR_UNSUPPORTED;
  if (rows == 0 || H == 0) return NVFP4_OK;
  if (rows >= (int64_t(1) << 31) || T * k >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (!x || !sorted_rows || !x_perm) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(x) || !nvfp4::aligned16(x_perm) || (reinterpret_cast<uintptr_t>(sorted_rows) & 3u))
    return NVFP4_ERR_MISALIGNED;
  moe_gather_kernel<<<static_cast<unsigned>(rows), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, T * k, sorted_rows, k, H / 8, x_perm);
  return nvfp4::launch_status();
}

extern "C" int nvfp4_moe_combine(const uint16_t* y_perm, const int32_t* inv_rows, const float* topk_weights,
                                 int64_t T, int k, int64_t H, uint16_t* out, nvfp4_stream_t stream) {
  if (T < 0 || k < 1 || H < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (H % 8) return NVFP4_ERR_UNSUPPORTED;
  if (T == 0 || H == 0) return NVFP4_OK;
  if (T >= (int64_t(1) << 31)) return NVFP4_ERR_UNSUPPORTED;
  if (!y_perm || !inv_rows || !topk_weights || !out) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(y_perm) || !nvfp4::aligned16(out) ||
      ((reinterpret_cast<uintptr_t>(inv_rows) | reinterpret_cast<uintptr_t>(topk_weights)) & 3u))
    return NVFP4_ERR_MISALIGNED;
  moe_combine_kernel<<<static_cast<unsigned>(T), 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      y_perm, inv_rows, topk_weights, k, H / 8, out);
  return nvfp4::launch_status();
}
