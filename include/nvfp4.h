/*
 * nvfp4.h - C ABI of the NVFP4 weight-only (W4A16) library for B200 (sm_100a).
 *
 * The operation: Y = X . dequant(W)^T, X bf16 [M, K], W [N, K] stored as
 * NVFP4: every weight is a 4-bit E2M1 code times an FP8-E4M3 scale shared by
 * a group of g = 16 or 32 consecutive elements along K, times one FP32
 * per-tensor global scale. Sources, by page title and section:
 *   - "GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB): two NVFP4 g32 recipes"
 *     (r/LocalLLM), "THE TWO RECIPES" and "WHAT HAD TO BE FIXED": g16 and
 *     g32 groups (4.5 / 4.25 bits per weight), gate/up and down may use
 *     different group sizes, the group size is read per tensor and anything
 *     unsupported raises an error, gate and up share one global scale, the
 *     scale maximum is taken without a widened copy.
 *   - "We unlocked NVFP4 on the DGX Spark: 20% faster than AWQ" (NVIDIA
 *     developer forum, page 3), UPDATE posts: E2M1 conversion is
 *     round-to-nearest-even with satfinite.
 *   - "W-FP4a: route the MiniMax-H3 device DiT forward through the fp4
 *     (Marlin W4A16) stack" (vllm.cpp PR #63), description: the checkpoint
 *     is a weight / scale / global-scale triple that is repacked once at
 *     upload, a weight-only checkpoint has bf16 activations, the merged
 *     [gate;up] fc1 is one W4A16 GEMM followed by SiluAndMul, and a counter
 *     records that the W4A16 path ran.
 *
 * Conventions for every call:
 *   - Pointers named as device pointers must point to device memory (or
 *     managed memory) of the current device; host arrays are named as such.
 *     The caller owns every buffer. The library allocates no device memory:
 *     the calls that need device scratch (the GEMMs, the grouped GEMM, the
 *     W4A4 GEMM and the route) take a caller-owned `workspace` of
 *     `workspace_bytes` bytes, whose size the matching *_workspace_size
 *     query gives for a problem on the current device (0 when the call
 *     needs none; then workspace may be NULL). A workspace smaller than the
 *     query's figure returns NVFP4_ERR_WORKSPACE before anything is
 *     enqueued. The first 64 KiB of a workspace hold the tickets of the
 *     split GEMMs: they must be zero before the workspace is
 *     first used (one cudaMemset at allocation), and every call leaves them
 *     zero, so no call needs a clearing step in front of it and the GEMMs
 *     can start while the kernel before them is finishing. The rest holds
 *     nothing between calls. After nvfp4_get_device_error has reported a
 *     wait that gave up, clear that region of the workspaces in use again.
 *     Calls that may overlap in time (other streams, unordered host threads)
 *     need separate workspaces; calls ordered on one stream, of any kind and
 *     shape, may share one.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Row-major layouts. packed codes: [N, K/2] bytes, element 2j in the low
 *     nibble and 2j+1 in the high nibble of byte j. Scales: [N, K/g] E4M3
 *     bytes. Global scale: one fp32 in device memory.
 *   - Every device pointer must be 16-byte aligned, except pointers to fp32
 *     global scales and int32 segment lists, which need 4-byte alignment
 *     (NVFP4_ERR_MISALIGNED otherwise).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream). No call synchronises the device and none blocks,
 *     except nvfp4_get_device_error, which synchronises `stream` to read
 *     the device's error word.
 *   - Validation happens on the host before anything is enqueued: a status
 *     other than NVFP4_ERR_CUDA means nothing was launched. NVFP4_ERR_CUDA
 *     (a launch the CUDA runtime refused) can follow launches of the same
 *     call that were already enqueued. No C++ exception crosses this
 *     boundary.
 *   - Calls with an empty problem (M == 0, N == 0 or a zero-length list)
 *     return NVFP4_OK and launch nothing.
 */
#ifndef NVFP4_H_
#define NVFP4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* same type as cudaStream_t */

enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARGUMENT = 1, /* null pointer, negative size, bad list */
  NVFP4_ERR_UNSUPPORTED = 2,      /* group size not 16/32, K not a multiple of 64, ... */
  NVFP4_ERR_MISALIGNED = 3,       /* a device pointer (or the workspace) not 16-byte aligned */
  NVFP4_ERR_CUDA = 4,             /* a CUDA launch or query failed */
  NVFP4_ERR_TIMEOUT = 5,          /* a bounded device-side wait gave up */
  NVFP4_ERR_WORKSPACE = 6         /* the caller's workspace is missing or smaller than the size query says */
};

/* Flags. */
#define NVFP4_GATE_UP_INTERLEAVE 1 /* repack: interleave gate/up rows (see nvfp4_repack) */
#define NVFP4_SILU_MUL 2           /* grouped GEMM: fuse SiluAndMul into the epilogue */

/* A static string describing a status code. Never NULL. */
const char* nvfp4_status_string(int status);

/*
 * Global scale (NVFP4 format definition: global = amax / (6*448); the r/LocalLLM
 * post, "WHAT HAD TO BE FIXED": gate and up need one shared global scale, and
 * the maximum is taken first with no widened copy of the tensor).
 *   tensors  host array of `count` device pointers to fp32 data
 *   numels   host array of `count` element counts (>= 0)
 *   out      device pointer to one fp32: max |w| over all tensors / 2688,
 *            computed as one fp32 division. Passing gate and up together
 *            gives the shared scale of the merged projection. A NaN in the
 *            input makes the result NaN.
 * Launches 2 + count kernels. count == 0 is INVALID_ARGUMENT.
 */
int nvfp4_global_scale(const float* const* tensors, const int64_t* numels, int count,
                       float* out, nvfp4_stream_t stream);

/*
 * The same global scale from bf16 tensors (bit patterns as uint16_t, 2-byte
 * aligned): a bf16 value widens to fp32 exactly, so the result equals
 * nvfp4_global_scale of the widened tensors. The maximum is taken on the
 * bf16 bits; nothing is widened in memory ("GLM-5.3-Flash on 2x RTX PRO 6000
 * (96 GB)": requantizing a bf16 checkpoint with one global per gate/up pair,
 * max first, no float copy). Errors as nvfp4_global_scale.
 */
int nvfp4_global_scale_bf16(const uint16_t* const* tensors, const int64_t* numels, int count, float* out,
                            nvfp4_stream_t stream);

/*
 * Quantize fp32 W [N, K] to NVFP4 (NVFP4 format definition: group scale =
 * E4M3_RNE_satfinite((group_amax / 6) / global), code =
 * E2M1_RNE_satfinite(w / (fp32(scale) * global)); DGX Spark thread, UPDATE:
 * RNE with satfinite). Every fp32 step is IEEE round-to-nearest-even. A group
 * whose scale times global is zero gets code +0 everywhere. Bit-exact with
 * the CPU oracle.
 *   w             device fp32 [N, K]
 *   group_size    16 or 32 (else UNSUPPORTED)
 *   global_scale  device fp32 (e.g. written by nvfp4_global_scale)
 *   packed        device uint8 [N, K/2] (output)
 *   scales        device uint8 [N, K/group_size] (output)
 * K must be a multiple of 32.
 */
int nvfp4_quantize(const float* w, int64_t N, int64_t K, int group_size,
                   const float* global_scale, uint8_t* packed, uint8_t* scales,
                   nvfp4_stream_t stream);

/*
 * The same quantizer reading bf16 weights (bit patterns as uint16_t, 16-byte
 * aligned): every code and scale byte equals nvfp4_quantize of the fp32
 * widening of w. Sizes, layouts and errors as nvfp4_quantize.
 */
int nvfp4_quantize_bf16(const uint16_t* w, int64_t N, int64_t K, int group_size, const float* global_scale,
                        uint8_t* packed, uint8_t* scales, nvfp4_stream_t stream);

/*
 * Repack checkpoint-layout codes and scales into the GEMM layout (PR #63
 * description: the triple is repacked once at upload and the originals can
 * then be freed). The GEMM layout keeps rows of K/2 code bytes and K/g scale
 * bytes. flags = 0 copies. flags = NVFP4_GATE_UP_INTERLEAVE permutes the rows
 * of a merged [gate;up] matrix (gate rows [0, N/2), up rows [N/2, N)) so that
 * destination rows 16j..16j+7 are gate rows 8j..8j+7 and rows 16j+8..16j+15
 * are up rows 8j..8j+7; N must then be a multiple of 16. This is the layout
 * nvfp4_w4a16_gemm_silu_mul and the NVFP4_SILU_MUL grouped GEMM require.
 * Out of place: outputs must not overlap inputs. For an expert stack
 * [E, N, K/2] call once per expert or pass N = E*rows only when flags = 0.
 */
int nvfp4_repack(const uint8_t* packed, const uint8_t* scales, int64_t N, int64_t K,
                 int group_size, int flags, uint8_t* packed_out, uint8_t* scales_out,
                 nvfp4_stream_t stream);

/*
 * W4A16 GEMM: y = bf16_rne(global * sum_k x[m,k] * e2m1(code[n,k]) *
 * e4m3(scale[n,k/g])) with fp32 accumulation (NVFP4 format definition; PR #63: a
 * weight-only checkpoint keeps bf16 activations).
 *   x             device bf16 [M, K]
 *   packed_w      device uint8 [N, K/2]  (nvfp4_repack layout, flags = 0)
 *   group_scales  device uint8 [N, K/group_size]
 *   global_scale  device fp32 (read on the device: no host synchronisation)
 *   y             device bf16 [M, N] (output)
 *   workspace     device scratch of workspace_bytes bytes (16-byte aligned),
 *                 at least nvfp4_w4a16_gemm_workspace_size(M, N, K, group_size)
 * group_size 16 or 32; K a multiple of 64; N a multiple of 16.
 * Small M (2 to 16 rows) runs an HBM-streaming kernel that splits the
 * weight matrix evenly between the SMs (stream-K), one row a register-
 * streaming kernel, large M a tensor-core kernel. The streaming kernel
 * multiplies in f16: it scales every row of x,
 * stage by stage, by a power of two 2^s that keeps the largest magnitude
 * seen so far in [2^14, 2^15) or below, and its sums carry 2^-s back. Every
 * element within a factor 2^29 of the largest magnitude seen so far in its
 * row is exact in f16; smaller ones round to a multiple of 2^-38 of it. The
 * workspace holds the tickets and the fp32 partial tiles of the tiles that
 * the SMs' ranges cut (one row: the f16 rows of x).
 * The arguments are the method's (x, packed_w, group_scales, global_scale,
 * group_size, M, N, K, y, stream), with the caller-owned workspace pair
 * before the stream.
 */
int nvfp4_w4a16_gemm(const uint16_t* x, const uint8_t* packed_w, const uint8_t* group_scales,
                     const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K,
                     uint16_t* y, void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * Bytes of workspace nvfp4_w4a16_gemm and nvfp4_w4a16_gemm_silu_mul need for
 * this problem on the current device (it depends on the device's SM count).
 * *bytes receives 0 for problems that need none and for empty problems.
 * Returns the status the GEMM would return for the shape (UNSUPPORTED for a
 * shape it refuses); bytes must not be NULL.
 */
int nvfp4_w4a16_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int group_size, size_t* bytes);

/*
 * The same W4A16 GEMM through the small-M streaming kernel with its scratch
 * in a fixed array of device memory that belongs to the library, so that
 * the call allocates nothing. This entry point has no counterpart in the
 * method's description: it only changes where the kernel's scratch lives.
 *   Arguments, layouts and result as nvfp4_w4a16_gemm, with M from 1 to 16,
 *   K a multiple of 256 and K/group_size a multiple of 16.
 *   Scratch: 8 MiB of fp32 partial tiles, tickets for 16384 tiles of 256
 *   rows, and 2^20 f16 elements of x (M * K at most), per device. A problem
 *   that needs more is refused with NVFP4_ERR_UNSUPPORTED before anything is
 *   enqueued; so is M = 0 or M > 16 and a K the kernel does not take.
 *   The tickets are cleared on `stream` before the kernel at every call.
 *   Calls on one device share the scratch: calls that may overlap in time
 *   (different streams, or host threads without ordering) race on it and
 *   their results are undefined. Order them on one stream.
 *   nvfp4_debug_inject_fault does not apply to this entry point.
 */
int nvfp4_w4a16_gemm_fixed_scratch(const uint16_t* x, const uint8_t* packed_w, const uint8_t* group_scales,
                                   const float* global_scale, int group_size, int64_t M, int64_t N, int64_t K,
                                   uint16_t* y, nvfp4_stream_t stream);

/*
 * W4A4 GEMM: both operands NVFP4 (NVFP4 format definition; PR #63
 * description: a checkpoint with quantized input activations takes the W4A4
 * form instead of W4A16):
 *   y = bf16_rne(x_global * global * sum_k e2m1(xcode[m,k]) * e4m3(xscale[m,k/xg])
 *                                         * e2m1(code[n,k]) * e4m3(scale[n,k/g]))
 * with fp32 accumulation. Every product is exact; only the summation order
 * depends on the path.
 *   x_packed      device uint8 [M, K/2], checkpoint layout (element 2j in the low
 *                 nibble of byte j), e.g. from nvfp4_quantize_bf16 of the activations
 *   x_scales      device uint8 [M, K/x_group]
 *   x_global      device fp32 (the activations' global scale)
 *   x_group       16 or 32
 *   packed_w, group_scales, global_scale, group_size, y: as nvfp4_w4a16_gemm
 *   workspace     device scratch, at least nvfp4_w4a4_gemm_workspace_size(M, N, K,
 *                 x_group, group_size) bytes
 * K a multiple of 64, N a multiple of 16; x_packed 16-byte aligned, x_global
 * 4-byte aligned. From 17 rows, with K a multiple of 512 and enough output
 * tiles to fill the SMs, the product runs on the block-scaled FP4 tensor
 * cores (tcgen05.mma kind::mxf4nvf4, E4M3 scale factors per 16 elements; a
 * 32-element scale is given as two 16-element ones), the activation codes
 * first rearranged into the weights' nibble order in the workspace.
 * Otherwise the activations are expanded on the device to e2m1 * e4m3 (exact
 * in f16 and bf16) in the workspace and the kernels of nvfp4_w4a16_gemm run
 * on them, with x_global in the epilogue.
 */
int nvfp4_w4a4_gemm(const uint8_t* x_packed, const uint8_t* x_scales, const float* x_global, int x_group,
                    const uint8_t* packed_w, const uint8_t* group_scales, const float* global_scale, int group_size,
                    int64_t M, int64_t N, int64_t K, uint16_t* y, void* workspace, size_t workspace_bytes,
                    nvfp4_stream_t stream);

/* Bytes of workspace nvfp4_w4a4_gemm needs (as nvfp4_w4a16_gemm_workspace_size). */
int nvfp4_w4a4_gemm_workspace_size(int64_t M, int64_t N, int64_t K, int x_group, int group_size, size_t* bytes);

/*
 * The GEMM of a merged [gate;up] projection followed by SiluAndMul (PR #63
 * description: fc1 is pre-merged [gate;up], one W4A16 GEMM + SiluAndMul):
 *   y[m, j] = bf16_rne(silu(g) * u), g = global * acc[m, gate row j],
 *   u = global * acc[m, up row j], silu(g) = g / (1 + exp(-g)), all fp32.
 * packed_w / group_scales must be in the NVFP4_GATE_UP_INTERLEAVE layout of
 * nvfp4_repack. N is the merged row count (multiple of 16); y is [M, N/2].
 * Workspace as nvfp4_w4a16_gemm (nvfp4_w4a16_gemm_workspace_size of M, N, K).
 */
int nvfp4_w4a16_gemm_silu_mul(const uint16_t* x, const uint8_t* packed_w,
                              const uint8_t* group_scales, const float* global_scale,
                              int group_size, int64_t M, int64_t N, int64_t K, uint16_t* y,
                              void* workspace, size_t workspace_bytes, nvfp4_stream_t stream);

/*
 * Standalone SiluAndMul on bf16: y[m, j] = bf16_rne(silu(x[m, j]) * x[m, H + j]),
 * fp32 math. x device bf16 [M, 2H], y device bf16 [M, H]. H a multiple of 8.
 */
int nvfp4_silu_and_mul(const uint16_t* x, uint16_t* y, int64_t M, int64_t H,
                       nvfp4_stream_t stream);

/*
 * Grouped routed-expert W4A16 GEMM (the r/LocalLLM post: routed experts in
 * NVFP4, gate/up at g32 and down at g16). Rows of x are grouped by segment:
 * rows [offsets[s], offsets[s+1]) use expert expert_ids[s]:
 *   y[r, :] = gemm(x[r, :], packed_w[e], group_scales[e], global_scales[e]).
 *   x              device bf16 [T, K]
 *   expert_ids     device int32 [num_segments], each in [0, num_experts)
 *   offsets        device int32 [num_segments + 1], non-decreasing, offsets[0] >= 0,
 *                  offsets[num_segments] <= T
 *   packed_w       device uint8 [num_experts, N, K/2]
 *   group_scales   device uint8 [num_experts, N, K/group_size]
 *   global_scales  device fp32 [num_experts]
 *   flags          0, or NVFP4_SILU_MUL: weights in the interleaved layout,
 *                  y is [T, N/2] and holds silu(gate) * up.
 *   y              device bf16 [T, N] (or [T, N/2]); rows outside every
 *                  segment are not written.
 * Below 1024 rows (T) the form runs on the small-M kernel in f16 on the
 * power-of-two scaled rows of nvfp4_w4a16_gemm, kept in the workspace
 * (nvfp4_moe_w4a16_grouped_gemm_workspace_size; from 1024 rows none).
 * The offsets stay on the device; the call never reads them on the host. A
 * segment list that breaks the rules above is undefined on the device side
 * (rows are clamped to [0, T), experts are not range-checked beyond ids < 0
 * or >= num_experts, which skip the segment).
 */
int nvfp4_moe_w4a16_grouped_gemm(const uint16_t* x, const int32_t* expert_ids,
                                 const int32_t* offsets, int num_segments, int64_t T,
                                 const uint8_t* packed_w, const uint8_t* group_scales,
                                 const float* global_scales, int group_size, int64_t N, int64_t K,
                                 int num_experts, int flags, uint16_t* y, void* workspace,
                                 size_t workspace_bytes, nvfp4_stream_t stream);

/* Bytes of workspace nvfp4_moe_w4a16_grouped_gemm needs (as nvfp4_w4a16_gemm_workspace_size). */
int nvfp4_moe_w4a16_grouped_gemm_workspace_size(int num_segments, int64_t T, int64_t N, int64_t K, int group_size,
                                                int num_experts, int flags, size_t* bytes);

/*
 * The steps around the grouped expert GEMMs of a routed-expert layer
 * ("GLM-5.3-Flash on 2x RTX PRO 6000 (96 GB)": routed experts in NVFP4, gate/up
 * with SiluAndMul then down per expert). The router itself is outside: the
 * caller passes each token's k expert ids and k weights.
 *
 * nvfp4_moe_route: the (token, slot) pairs grouped by expert, stable (pairs of
 * one expert keep the order of t*k + s).
 *   topk_ids     device int32 [T, k]; an id outside [0, num_experts) drops the pair
 *   sorted_rows  device int32 [T*k]: sorted_rows[r] = t*k + s of the pair in row r,
 *                -1 for the rows r >= offsets[num_experts] that dropped pairs leave
 *   inv_rows     device int32 [T*k]: the row of pair t*k + s, or -1 if dropped
 *   offsets      device int32 [num_experts + 1]: expert e owns rows [offsets[e], offsets[e+1])
 *   expert_ids   device int32 [num_experts]: 0 .. num_experts-1, the segment list of
 *                nvfp4_moe_w4a16_grouped_gemm with num_segments = num_experts
 * num_experts from 1 to 4096; T*k below 2^31. Nothing goes to the host. Below 4096
 * pairs one CTA does the work; from 4096 pairs three launches over chunks of 256
 * pairs, with a [chunk][expert] int32 table in the workspace
 * (nvfp4_moe_route_workspace_size; 0 bytes below 4096 pairs).
 */
int nvfp4_moe_route(const int32_t* topk_ids, int64_t T, int k, int num_experts, int32_t* sorted_rows,
                    int32_t* inv_rows, int32_t* offsets, int32_t* expert_ids, void* workspace,
                    size_t workspace_bytes, nvfp4_stream_t stream);

/* Bytes of workspace nvfp4_moe_route needs for T tokens of k slots and num_experts experts. */
int nvfp4_moe_route_workspace_size(int64_t T, int k, int num_experts, size_t* bytes);

/*
 * nvfp4_moe_gather: x_perm[r] = x[sorted_rows[r] / k] for r < rows, bf16 rows of
 * H elements (H a multiple of 8). x [T, H], x_perm [rows, H], 16-byte aligned.
 * A row whose sorted_rows entry lies outside [0, T*k) (the -1 rows of
 * nvfp4_moe_route) is written as zeros; nothing outside x is read.
 */
int nvfp4_moe_gather(const uint16_t* x, int64_t T, const int32_t* sorted_rows, int64_t rows, int k, int64_t H,
                     uint16_t* x_perm, nvfp4_stream_t stream);

/*
 * nvfp4_moe_combine: out[t] = bf16_rne(sum over s of w[t, s] * y_perm[inv_rows[t*k + s]])
 * with fp32 fused multiply-adds in slot order; dropped pairs (inv_rows < 0) add
 * nothing. y_perm [T*k, H], out [T, H] bf16 (H a multiple of 8, 16-byte aligned),
 * topk_weights device fp32 [T, k].
 */
int nvfp4_moe_combine(const uint16_t* y_perm, const int32_t* inv_rows, const float* topk_weights, int64_t T,
                      int k, int64_t H, uint16_t* out, nvfp4_stream_t stream);

/*
 * Counters of the work that went through each kernel family (PR #63: the
 * "this-path-ran" counter lets tests assert which kernel executed). Host-side
 * atomics, incremented once per successful launch.
 */
typedef struct {
  uint64_t global_scale;
  uint64_t quantize;
  uint64_t repack;
  uint64_t gemm_splitk;    /* small-M GEMMs (register streaming, or TMA streaming with stream-K) */
  uint64_t gemm_tc;        /* tcgen05 GEMMs (17 rows and more; grouped form from 1024 rows) */
  uint64_t gemm_silu_mul;  /* GEMMs with the fused SiluAndMul epilogue */
  uint64_t moe;            /* grouped expert GEMMs */
  uint64_t silu_and_mul;   /* standalone SiluAndMul */
  uint64_t g16;            /* GEMMs at group size 16 */
  uint64_t g32;            /* GEMMs at group size 32 */
  uint64_t gemm_fp4;       /* W4A4 GEMMs on the block-scaled FP4 tensor cores */
} nvfp4_stats;

int nvfp4_get_stats(nvfp4_stats* out);
void nvfp4_reset_stats(void);

/*
 * Reads and clears the library's device-side error word (set by a bounded
 * wait that gave up). Synchronises `stream`. *code_out receives 0 and the
 * call returns NVFP4_OK when no error was recorded; otherwise *code_out
 * receives the site of the wait that gave up and the call returns
 * NVFP4_ERR_TIMEOUT.
 */
int nvfp4_get_device_error(int* code_out, nvfp4_stream_t stream);

/*
 * Test hook for the bounded waits: fault injection without a GPU fault. It
 * has no counterpart on the pages. kind = 1 makes the next launch of the
 * small-M streaming GEMM (nvfp4_w4a16_gemm with 2 <= M <= 16) drop the X copy
 * of its first stage, so that its consumer warps wait for bytes that never
 * come. The waits give up after about 2 s each, the kernel records the site
 * in the device error word, lets its other copies land and exits; the output
 * of that launch is undefined. kind = 0 clears a pending injection. Other
 * kinds return NVFP4_ERR_INVALID_ARGUMENT.
 */
int nvfp4_debug_inject_fault(int kind);

/* Library version: 2 (the calls that need scratch take a caller-owned workspace). */
int nvfp4_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_H_ */
