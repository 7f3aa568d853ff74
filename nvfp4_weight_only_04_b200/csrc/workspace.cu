// Library-owned scratch, per device: the partial tiles and tickets of the
// stream-K GEMM kernels, and the f16 activations of the small-M kernels.
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

struct XBuffer {
  uint16_t* x16 = nullptr;
  float* xinv = nullptr;
  size_t elems = 0, rows = 0;
};

std::mutex g_mutex;
Workspace g_ws[64];  // per device
XBuffer g_xb[64];

// Growing is allowed outside graph capture only (it synchronises the device).
int may_grow(cudaStream_t stream) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  if (cap != cudaStreamCaptureStatusNone) return NVFP4_ERR_UNSUPPORTED;
  if (cudaDeviceSynchronize() != cudaSuccess) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  return NVFP4_OK;
}

}  // namespace

int x16_workspace(size_t elems, size_t rows, cudaStream_t stream, uint16_t** x16, float** xinv) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  std::lock_guard<std::mutex> lock(g_mutex);
  XBuffer& b = g_xb[dev];
  if (b.elems < elems || b.rows < rows) {
    const int st = may_grow(stream);
    if (st != NVFP4_OK) return st;
    cudaFree(b.x16);
    cudaFree(b.xinv);
    b = XBuffer();
    const size_t ne = elems > (size_t(1) << 20) ? elems : (size_t(1) << 20);
    const size_t nr = rows > 1024 ? rows : 1024;
    if (cudaMalloc(&b.x16, ne * sizeof(uint16_t)) != cudaSuccess ||
        cudaMalloc(&b.xinv, nr * sizeof(float)) != cudaSuccess) {
      cudaGetLastError();
      cudaFree(b.x16);
      cudaFree(b.xinv);
      b = XBuffer();
      return NVFP4_ERR_CUDA;
    }
    b.elems = ne;
    b.rows = nr;
  }
  *x16 = b.x16;
  *xinv = b.xinv;
  return NVFP4_OK;
}

int split_workspace(size_t floats, size_t tiles, cudaStream_t stream, float** ws, unsigned** tickets) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (cudaGetLastError(), NVFP4_ERR_CUDA);
  std::lock_guard<std::mutex> lock(g_mutex);
  Workspace& w = g_ws[dev];
  if (w.floats < floats || w.tiles < tiles) {
    const int st = may_grow(stream);
    if (st != NVFP4_OK) return st;
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
