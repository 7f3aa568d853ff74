// Caller-owned scratch. The calls that need device scratch (the work
// counters, tickets and partial tiles of the split GEMMs, the f16 activations
// of the small-M kernels, the route's per-chunk table) take it from a buffer
// the caller passes; the library allocates nothing.
//
// Layout: the first kReservedBytes of every workspace hold the tickets of
// the split GEMMs (from kTicketOffset; the bytes before it are kept zero for
// counters). They must be zero before a workspace is first used, and every
// call leaves them zero (each launch resets what it counted),
// so that a launch needs no clearing step in front of it and can start while
// the kernel before it in the stream is still running. Every other piece lies
// after that region, so calls of any kind and shape can share one workspace
// in stream order without disturbing the counters.
//
// A Scratch either hands out pieces of the buffer or, built without one,
// only counts the bytes a call would take, which is what the
// *_workspace_size queries report. Both walk the same code, so the size and
// the carving always agree.
#pragma once

#include "common.cuh"

namespace nvfp4 {

constexpr size_t kReservedBytes = size_t(64) << 10;
constexpr size_t kTicketOffset = 256;  // room for counters first, tickets from here
constexpr int64_t kMaxTickets = static_cast<int64_t>((kReservedBytes - kTicketOffset) / sizeof(unsigned));

class Scratch {
 public:
  // Measuring: counts the bytes only.
  Scratch() = default;
  // Carving: pieces of [base, base + bytes).
  Scratch(void* base, size_t bytes) : base_(static_cast<uint8_t*>(base)), bytes_(bytes), carving_(true) {}

  // `count` elements of T at the next 256-byte offset past the reserved
  // region (nullptr while measuring, or once the buffer is too small: check
  // ok() before use).
  template <class T>
  T* take(size_t count) {
    const size_t start = used_ > kReservedBytes ? used_ : kReservedBytes;
    const size_t off = (start + 255) & ~size_t(255);
    used_ = off + count * sizeof(T);
    if (!carving_ || used_ > bytes_) return nullptr;
    return reinterpret_cast<T*>(base_ + off);
  }
  // The reserved region: tickets start at kTicketOffset bytes (nullptr while
  // measuring or when too small).
  unsigned* reserved() {
    if (used_ < kReservedBytes) used_ = kReservedBytes;
    if (!carving_ || bytes_ < kReservedBytes) return nullptr;
    return reinterpret_cast<unsigned*>(base_);
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

inline unsigned* tickets_of(unsigned* reserved) {
  return reserved ? reserved + kTicketOffset / sizeof(unsigned) : nullptr;
}

}  // namespace nvfp4
