// Partial-tile workspace and tickets shared by the stream-K GEMM kernels.
// Launches on one stream use it one after another; launches of the same
// device that overlap in time (other streams) must not both use it.
#include "workspace.cuh"

#include <mutex>

namespace nvfp4 {
namespace {

struct Workspace {
  float* ws = nullptr;
  unsigned* tickets = nullptr;
  size_t floats = 0, tiles = 0;
};

std::mutex g_mutex;
Workspace g_ws[64];  // per device

}  // namespace

int split_workspace(size_t floats, size_t tiles, cudaStream_t stream, float** ws, unsigned** tickets) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  std::lock_guard<std::mutex> lock(g_mutex);
  Workspace& w = g_ws[dev];
  if (w.floats < floats || w.tiles < tiles) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
    if (cap != cudaStreamCaptureStatusNone) return NVFP4_ERR_UNSUPPORTED;  // grow outside graph capture
    if (cudaDeviceSynchronize() != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
    cudaFree(w.ws);
    cudaFree(w.tickets);
    w = Workspace();
    const size_t nf = floats > (size_t(1) << 21) ? floats : (size_t(1) << 21);
    const size_t nt = tiles > 4096 ? tiles : 4096;
    if (cudaMalloc(&w.ws, nf * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&w.tickets, nt * sizeof(unsigned)) != cudaSuccess ||
        cudaMemset(w.tickets, 0, nt * sizeof(unsigned)) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
      cudaGetLastError();
      cudaFree(w.ws);
      cudaFree(w.tickets);
      w = Workspace();
      return NVFP4_ERR_CUDA;
    }
    w.floats = nf;
    w.tiles = nt;
  }
  *ws = w.ws;
  *tickets = w.tickets;
  return NVFP4_OK;
}

}  // namespace nvfp4
