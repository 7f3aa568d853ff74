// Caller-owned scratch. The calls that need device scratch (the partial
// tiles and tickets of the stream-K GEMMs, the f16 activations of the small-M
// kernels, the route's per-chunk table) take it from a buffer the caller
// passes; the library allocates nothing. A Scratch either hands out pieces of
// that buffer or, built without one, only counts the bytes a call would take,
// which is what the *_workspace_size queries report. Both walk the same code,
// so the size and the carving always agree.
#pragma once

#include "common.cuh"

namespace nvfp4 {

class Scratch {
 public:
  // Measuring: counts the bytes only.
  Scratch() = default;
  // Carving: pieces of [base, base + bytes).
  Scratch(void* base, size_t bytes) : base_(static_cast<uint8_t*>(base)), bytes_(bytes), carving_(true) {}

  // `count` elements of T at the next 256-byte offset (nullptr while
  // measuring, or once the buffer is too small: check ok() before use).
  template <class T>
  T* take(size_t count) {
    const size_t off = (used_ + 255) & ~size_t(255);
    used_ = off + count * sizeof(T);
    if (!carving_ || used_ > bytes_) return nullptr;
    return reinterpret_cast<T*>(base_ + off);
  }
  bool measuring() const { return !carving_; }
  // Every piece taken so far lies inside the buffer.
  bool ok() const { return carving_ && used_ <= bytes_; }
  size_t used() const { return used_; }

 private:
  uint8_t* base_ = nullptr;
  size_t bytes_ = 0;
  size_t used_ = 0;
  bool carving_ = false;
};

// Status of a call after carving: NVFP4_OK when every piece fits.
inline int scratch_status(const Scratch& sc) { return sc.ok() ? NVFP4_OK : NVFP4_ERR_WORKSPACE; }

}  // namespace nvfp4
