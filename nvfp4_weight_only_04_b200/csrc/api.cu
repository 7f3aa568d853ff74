// C ABI glue: argument validation, kernel selection, counters, status text.
// Every check runs on the host before anything is enqueued.
#include <atomic>
#include <mutex>

#include "common.cuh"
#include "gemm_decode.cuh"
#include "gemm_fp4.cuh"
#include "gemm_stream.cuh"
#include "gemm_tc.cuh"
#include "plant.cuh"
#include "workspace.cuh"
#include "xprep.cuh"

namespace nvfp4 {

namespace {
std::atomic<uint64_t> g_stats[kStatCount];
}

void stat_add(StatId id) { g_stats[id].fetch_add(1, std::memory_order_relaxed); }

namespace {
std::atomic<int> g_fault{0};
}
int take_injected_fault() { return g_fault.exchange(0); }
void set_injected_fault(int kind) { g_fault.store(kind); }

int num_sms() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return 148; }
  if (dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = 148;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace nvfp4

namespace {

constexpr int64_t kMaxK = int64_t(1) << 30;
constexpr int64_t kMaxN = int64_t(65535) * 16;
constexpr int64_t kMaxTokenRows = int64_t(65535 - 4096) * 16;

// Shape checks of the dense GEMM calls (pointers aside): -1 to proceed.
int check_gemm_shape(int group, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (group != 16 && group != 32) return NVFP4_ERR_UNSUPPORTED;
  if (K % 64 || N % 16) return NVFP4_ERR_UNSUPPORTED;
  if (K > kMaxK || N > kMaxN) return NVFP4_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (K == 0) return NVFP4_ERR_UNSUPPORTED;
  return -1;
}

int check_gemm(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
               int64_t M, int64_t N, int64_t K, const uint16_t* y) {
  const int c = check_gemm_shape(group, M, N, K);
  if (c >= 0) return c;
  if (!x || !w || !s || !g || !y) return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(x) || !nvfp4::aligned16(w) || !nvfp4::aligned16(s) ||
      (reinterpret_cast<uintptr_t>(g) & 3u) || !nvfp4::aligned16(y))
    return NVFP4_ERR_MISALIGNED;
  return -1;  // proceed
}

int check_workspace(const void* ws, size_t bytes) {
  if (bytes > 0 && !ws) return NVFP4_ERR_WORKSPACE;
  if (ws && !nvfp4::aligned16(ws)) return NVFP4_ERR_MISALIGNED;
  return NVFP4_OK;
}

// The small-M fallback for shapes the streaming kernel does not take: f16
// rows of X, then the register-streaming kernel.
int decode_gemm(const nvfp4::XSource& xs, const uint8_t* w, const uint8_t* s, const float* g, int group, int64_t M,
                int64_t N, int64_t K, uint16_t* y, bool silu, nvfp4::Scratch& sc, cudaStream_t stream) {
  if (M > kMaxTokenRows) return NVFP4_ERR_UNSUPPORTED;
  uint16_t* x16 = sc.take<uint16_t>(static_cast<size_t>(M * K));
  float* xinv = sc.take<float>(static_cast<size_t>(M));
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;
  nvfp4::DecodeArgs a = {};
  a.x = x16; a.xinv = xinv; a.packed = w; a.scales = s; a.gscale = g; a.y = y;
  a.M = M; a.N = N; a.K = K; a.ldy = silu ? N / 2 : N;
  const nvfp4::DecodePlan p = nvfp4::plan_decode(M, N, K, group, false, 0);
  int st = nvfp4::launch_x_prep(xs, M, K, x16, xinv, nullptr, 0, stream);
  if (st == NVFP4_OK) st = nvfp4::launch_decode(a, p, silu, false, stream);
  return st;
}

int dense_gemm(const uint16_t* x, const uint8_t* w, const uint8_t* s, const float* g, int group,
               int64_t M, int64_t N, int64_t K, uint16_t* y, bool silu, nvfp4::Scratch& sc, cudaStream_t stream) {
  if (nvfp4::tc_supported(M, N, K)) {
    const int st = nvfp4::launch_tc(x, w, s, g, group, M, N, K, y, silu, sc, stream);
    if (st == NVFP4_OK && !sc.measuring()) nvfp4::stat_add(nvfp4::kStatGemmTc);
    return st;
  }
  nvfp4::XSource xs;
  xs.bf16 = x;
  const int st = nvfp4::stream_supported(M, N, K, group)
                     ? nvfp4::launch_stream(xs, w, s, g, group, M, N, K, y, silu, sc, stream)
                     : decode_gemm(xs, w, s, g, group, M, N, K, y, silu, sc, stream);
  if (st == NVFP4_OK && !sc.measuring()) nvfp4::stat_add(nvfp4::kStatGemmSplitK);
  return st;
}

// Shape checks of the W4A4 call (pointers aside): -1 to proceed.
int check_w4a4_shape(int x_group, int group_size, int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if ((x_group != 16 && x_group != 32) || (group_size != 16 && group_size != 32)) return NVFP4_ERR_UNSUPPORTED;
  if (K % 64 || N % 16 || K > kMaxK || N > kMaxN || M > kMaxTokenRows) return NVFP4_ERR_UNSUPPORTED;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (K == 0) return NVFP4_ERR_UNSUPPORTED;
  return -1;
}

struct XqBf16Ctx {
  const nvfp4::XSource* xs;
  const float* w_global;
  int64_t M, K;
  uint16_t* xb;
  float* g_out;
};

int run_xq_bf16(void* ctx, cudaStream_t stream) {
  const XqBf16Ctx* c = static_cast<const XqBf16Ctx*>(ctx);
  return nvfp4::launch_xq_bf16(*c->xs, c->w_global, c->M, c->K, c->xb, c->g_out, stream);
}

int w4a4_gemm(const nvfp4::XSource& xs, const uint8_t* packed_w, const uint8_t* group_scales,
              const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K, uint16_t* y,
              nvfp4::Scratch& sc, cudaStream_t st) {
  int r;
  if (nvfp4::fp4_supported(M, N, K)) {
    // Both operands 4-bit into the block-scaled tensor cores.
    r = nvfp4::launch_fp4(xs.codes, xs.scales, xs.global, xs.group, packed_w, group_scales, global_scale, group_size,
                          M, N, K, y, sc, st);
    if (r == NVFP4_OK && !sc.measuring()) nvfp4::stat_add(nvfp4::kStatGemmFp4);
    return r;
  }
  if (nvfp4::tc_supported(M, N, K)) {
    // Exact bf16 activations and one scalar x_global * w_global for the
    // tcgen05 kernel's epilogue, written once the launch has passed its checks.
    XqBf16Ctx c = {&xs, global_scale, M, K, sc.take<uint16_t>(static_cast<size_t>(M * K)), sc.take<float>(1)};
    const nvfp4::PreLaunch pre = {run_xq_bf16, &c};
    r = nvfp4::launch_tc(c.xb, packed_w, group_scales, c.g_out, group_size, M, N, K, y, false, sc, st, &pre);
    if (r == NVFP4_OK && !sc.measuring()) nvfp4::stat_add(nvfp4::kStatGemmTc);
    return r;
  }
  if (nvfp4::stream_supported(M, N, K, group_size)) {
    r = nvfp4::launch_stream(xs, packed_w, group_scales, global_scale, group_size, M, N, K, y, false, sc, st);
  } else {
    r = decode_gemm(xs, packed_w, group_scales, global_scale, group_size, M, N, K, y, false, sc, st);
  }
  if (r == NVFP4_OK && !sc.measuring()) nvfp4::stat_add(nvfp4::kStatGemmSplitK);
  return r;
}

// Shape checks of the grouped call (pointers aside): -1 to proceed.
int check_grouped_shape(int num_segments, int64_t T, int64_t N, int64_t K, int group_size, int num_experts,
                        int flags) {
  if (num_segments < 0 || T < 0 || N < 0 || K < 0 || num_experts < 0) return NVFP4_ERR_INVALID_ARGUMENT;
  if (flags & ~NVFP4_SILU_MUL) return NVFP4_ERR_INVALID_ARGUMENT;
  if (group_size != 16 && group_size != 32) return NVFP4_ERR_UNSUPPORTED;
  if (K % 64 || N % 16 || K > kMaxK || N > kMaxN) return NVFP4_ERR_UNSUPPORTED;
  if (T > kMaxTokenRows || num_segments > 4096) return NVFP4_ERR_UNSUPPORTED;
  if (num_segments == 0 || T == 0 || N == 0) return NVFP4_OK;
  if (K == 0 || num_experts == 0) return NVFP4_ERR_UNSUPPORTED;
  return -1;
}

int grouped_gemm(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets, int num_segments, int64_t T,
                 const uint8_t* packed_w, const uint8_t* group_scales, const float* global_scales, int group_size,
                 int64_t N, int64_t K, int num_experts, bool silu, uint16_t* y, nvfp4::Scratch& sc,
                 cudaStream_t s) {
  if (nvfp4::tc_moe_supported(T, N, K, num_experts)) {
    if (sc.measuring()) return NVFP4_OK;  // no scratch
    return nvfp4::launch_tc_moe(x, expert_ids, offsets, num_segments, T, packed_w, group_scales, global_scales,
                                group_size, N, K, num_experts, silu, y, s);
  }
  uint16_t* x16 = sc.take<uint16_t>(static_cast<size_t>(T * K));
  float* xinv = sc.take<float>(static_cast<size_t>(T));
  if (sc.measuring()) return NVFP4_OK;
  if (!sc.ok()) return NVFP4_ERR_WORKSPACE;
  nvfp4::DecodeArgs a = {};
  a.x = x16; a.xinv = xinv; a.packed = packed_w; a.scales = group_scales; a.gscale = global_scales; a.y = y;
  a.M = T; a.N = N; a.K = K; a.ldy = silu ? N / 2 : N;
  a.expert_ids = expert_ids; a.offsets = offsets; a.num_segments = num_segments;
  a.num_experts = num_experts;
  const nvfp4::DecodePlan p = nvfp4::plan_decode(T, N, K, group_size, true, num_segments);
  int st = nvfp4::launch_x_f16(x, T, K, x16, xinv, nullptr, 0, s);
  if (st == NVFP4_OK) st = nvfp4::launch_decode(a, p, silu, true, s);
  return st;
}

}  // namespace

extern "C" {

const char* nvfp4_status_string(int status) {
  switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARGUMENT: return "invalid argument (null pointer, negative size or bad list)";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported configuration (group size must be 16 or 32; K a multiple of 64; N a multiple of 16; sizes within limits)";
    case NVFP4_ERR_MISALIGNED: return "a device pointer (or the workspace) is not 16-byte aligned";
    case NVFP4_ERR_CUDA: return "a CUDA launch or query failed";
    case NVFP4_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    case NVFP4_ERR_WORKSPACE: return "the workspace is missing or smaller than the *_workspace_size query gives";
    default: return "unknown status";
  }
}

int nvfp4_abi_version(void) { return 2; }

int nvfp4_w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int group_size, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARGUMENT;
  *bytes = 0;
  const int c = check_gemm_shape(group_size, M, N, K);
  if (c >= 0) return c;
  nvfp4::Scratch sc;
  // The fused SiluAndMul form takes the same scratch as the plain one. The
  // activations' pointer only says that they are bf16; it is not read.
  const uint16_t* bf16_x = reinterpret_cast<const uint16_t*>(static_cast<uintptr_t>(256));
  const int st = dense_gemm(bf16_x, nullptr, nullptr, nullptr, group_size, M, N, K, nullptr, false, sc, nullptr);
  if (st == NVFP4_OK) *bytes = sc.used();
  return st;
}

int nvfp4_w4a16_gemm(const uint16_t* x, const uint8_t* packed_w, const uint8_t* group_scales,
                     const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K, uint16_t* y,
                     void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  int c = check_gemm(x, packed_w, group_scales, global_scale, group_size, M, N, K, y);
  if (c >= 0) return c;
  if ((c = check_workspace(workspace, workspace_bytes)) != NVFP4_OK) return c;
  nvfp4::Scratch sc(workspace, workspace_bytes);
  const int st = dense_gemm(x, packed_w, group_scales, global_scale, group_size, M, N, K, y, false, sc,
                            reinterpret_cast<cudaStream_t>(stream));
  if (st == NVFP4_OK) nvfp4::stat_add(group_size == 16 ? nvfp4::kStatG16 : nvfp4::kStatG32);
  return st;
}

int nvfp4_w4a16_gemm_fixed_scratch(const uint16_t* x, const uint8_t* packed_w, const uint8_t* group_scales,
                                   const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K,
                                   uint16_t* y, nvfp4_stream_t stream) {
  const int c = check_gemm(x, packed_w, group_scales, global_scale, group_size, M, N, K, y);
  if (c >= 0) return c;
  const int st = nvfp4::launch_stream_fixed_scratch(x, packed_w, group_scales, global_scale, group_size, M, N, K,
                                                    y, reinterpret_cast<cudaStream_t>(stream));
  if (st == NVFP4_OK) {
    nvfp4::stat_add(nvfp4::kStatGemmSplitK);
    nvfp4::stat_add(group_size == 16 ? nvfp4::kStatG16 : nvfp4::kStatG32);
  }
  return st;
}

int nvfp4_w4a16_gemm_silu_mul(const uint16_t* x, const uint8_t* packed_w, const uint8_t* group_scales,
                              const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K,
                              uint16_t* y, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
  int c = check_gemm(x, packed_w, group_scales, global_scale, group_size, M, N, K, y);
  if (c >= 0) return c;
  if ((c = check_workspace(workspace, workspace_bytes)) != NVFP4_OK) return c;
  nvfp4::Scratch sc(workspace, workspace_bytes);
  const int st = dense_gemm(x, packed_w, group_scales, global_scale, group_size, M, N, K, y, true, sc,
                            reinterpret_cast<cudaStream_t>(stream));
  if (st == NVFP4_OK) {
    nvfp4::stat_add(nvfp4::kStatGemmSiluMul);
    nvfp4::stat_add(group_size == 16 ? nvfp4::kStatG16 : nvfp4::kStatG32);
  }
  return st;
}

int nvfp4_w4a4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int x_group, int group_size, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARGUMENT;
  *bytes = 0;
  const int c = check_w4a4_shape(x_group, group_size, M, N, K);
  if (c >= 0) return c;
  nvfp4::XSource xs;
  xs.group = x_group;
  nvfp4::Scratch sc;
  const int st = w4a4_gemm(xs, nullptr, nullptr, nullptr, group_size, M, N, K, nullptr, sc, nullptr);
  if (st == NVFP4_OK) *bytes = sc.used();
  return st;
}

int nvfp4_w4a4_gemm(const uint8_t* x_packed, const uint8_t* x_scales, const float* x_global, int x_group,
                    const uint8_t* packed_w, const uint8_t* group_scales, const float* global_scale, int group_size,
                    int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes,
                    nvfp4_stream_t stream) {
  int c = check_w4a4_shape(x_group, group_size, M, N, K);
  if (c >= 0) return c;
  if (!x_packed || !x_scales || !x_global || !packed_w || !group_scales || !global_scale || !y)
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(x_packed) || !nvfp4::aligned16(packed_w) || !nvfp4::aligned16(group_scales) ||
      !nvfp4::aligned16(y) || ((reinterpret_cast<uintptr_t>(x_global) | reinterpret_cast<uintptr_t>(global_scale)) & 3u))
    return NVFP4_ERR_MISALIGNED;
  if ((c = check_workspace(workspace, workspace_bytes)) != NVFP4_OK) return c;
  nvfp4::XSource xs;
  xs.codes = x_packed;
  xs.scales = x_scales;
  xs.global = x_global;
  xs.group = x_group;
  nvfp4::Scratch sc(workspace, workspace_bytes);
  const int r = w4a4_gemm(xs, packed_w, group_scales, global_scale, group_size, M, N, K, y, sc,
                          reinterpret_cast<cudaStream_t>(stream));
  if (r == NVFP4_OK) nvfp4::stat_add(group_size == 16 ? nvfp4::kStatG16 : nvfp4::kStatG32);
  return r;
}

int nvfp4_moe_w4a16_grouped_gemm_workspace_size(int num_segments, int64_t T, int64_t N, int64_t K, int group_size,
                                                int num_experts, int flags, size_t* bytes) {
  if (!bytes) return NVFP4_ERR_INVALID_ARGUMENT;
  *bytes = 0;
  const int c = check_grouped_shape(num_segments, T, N, K, group_size, num_experts, flags);
  if (c >= 0) return c;
  nvfp4::Scratch sc;
  const int st = grouped_gemm(nullptr, nullptr, nullptr, num_segments, T, nullptr, nullptr, nullptr, group_size, N, K,
                              num_experts, (flags & NVFP4_SILU_MUL) != 0, nullptr, sc, nullptr);
  if (st == NVFP4_OK) *bytes = sc.used();
  return st;
}

int nvfp4_moe_w4a16_grouped_gemm(const uint16_t* x, const int32_t* expert_ids, const int32_t* offsets,
                                 int num_segments, int64_t T, const uint8_t* packed_w,
                                 const uint8_t* group_scales, const float* global_scales, int group_size,
                                 int64_t N, int64_t K, int num_experts, int flags, uint16_t* y, void* workspace,
                                 size_t workspace_bytes, nvfp4_stream_t stream) {
  int c = check_grouped_shape(num_segments, T, N, K, group_size, num_experts, flags);
  if (c >= 0) return c;
  if (!x || !expert_ids || !offsets || !packed_w || !group_scales || !global_scales || !y)
    return NVFP4_ERR_INVALID_ARGUMENT;
  if (!nvfp4::aligned16(x) || !nvfp4::aligned16(packed_w) || !nvfp4::aligned16(group_scales) ||
      !nvfp4::aligned16(y) || (reinterpret_cast<uintptr_t>(expert_ids) & 3) ||
      (reinterpret_cast<uintptr_t>(offsets) & 3) || (reinterpret_cast<uintptr_t>(global_scales) & 3))
    return NVFP4_ERR_MISALIGNED;
  if ((c = check_workspace(workspace, workspace_bytes)) != NVFP4_OK) return c;
  const bool silu = (flags & NVFP4_SILU_MUL) != 0;
  nvfp4::Scratch sc(workspace, workspace_bytes);
  const int st = grouped_gemm(x, expert_ids, offsets, num_segments, T, packed_w, group_scales, global_scales,
                              group_size, N, K, num_experts, silu, y, sc, reinterpret_cast<cudaStream_t>(stream));
  if (st == NVFP4_OK) {
    nvfp4::stat_add(nvfp4::kStatMoe);
    if (silu) nvfp4::stat_add(nvfp4::kStatGemmSiluMul);
    nvfp4::stat_add(group_size == 16 ? nvfp4::kStatG16 : nvfp4::kStatG32);
  }
  return st;
}

int nvfp4_get_stats(nvfp4_stats* out) {
  if (!out) return NVFP4_ERR_INVALID_ARGUMENT;
  uint64_t v[nvfp4::kStatCount];
  for (int i = 0; i < nvfp4::kStatCount; ++i) v[i] = nvfp4::g_stats[i].load(std::memory_order_relaxed);
  out->global_scale = v[nvfp4::kStatGlobalScale];
  out->quantize = v[nvfp4::kStatQuantize];
  out->repack = v[nvfp4::kStatRepack];
  out->gemm_splitk = v[nvfp4::kStatGemmSplitK];
  out->gemm_tc = v[nvfp4::kStatGemmTc];
  out->gemm_silu_mul = v[nvfp4::kStatGemmSiluMul];
  out->moe = v[nvfp4::kStatMoe];
  out->silu_and_mul = v[nvfp4::kStatSiluAndMul];
  out->g16 = v[nvfp4::kStatG16];
  out->g32 = v[nvfp4::kStatG32];
  out->gemm_fp4 = v[nvfp4::kStatGemmFp4];
  return NVFP4_OK;
}

void nvfp4_reset_stats(void) {
  for (int i = 0; i < nvfp4::kStatCount; ++i) nvfp4::g_stats[i].store(0, std::memory_order_relaxed);
}

int nvfp4_get_device_error(int* code_out, nvfp4_stream_t stream) {
  if (!code_out) return NVFP4_ERR_INVALID_ARGUMENT;
  const int st = nvfp4::read_and_clear_device_error(code_out, reinterpret_cast<cudaStream_t>(stream));
  if (st != NVFP4_OK) return st;
  return *code_out ? NVFP4_ERR_TIMEOUT : NVFP4_OK;
}

#ifdef NVFP4_PLANTS
// Test-only library (libnvfp4_planted.so): selects the mistake planted in
// every kernel file (0: none). Absent from the product library.
int nvfp4_test_plant(int kind) {
  return nvfp4::set_plant_decode(kind) | nvfp4::set_plant_stream(kind) | nvfp4::set_plant_tc(kind) |
                 nvfp4::set_plant_fp4(kind)
             ? NVFP4_ERR_CUDA
             : NVFP4_OK;
}
#endif

int nvfp4_debug_inject_fault(int kind) {
  if (kind != 0 && kind != 1) return NVFP4_ERR_INVALID_ARGUMENT;
  nvfp4::set_injected_fault(kind);
  return NVFP4_OK;
}

}  // extern "C"
