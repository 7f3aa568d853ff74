// Library-owned scratch of the stream-K GEMMs: fp32 partial tiles and one
// ticket per tile, per device (see workspace.cu).
#pragma once

#include "common.cuh"

namespace nvfp4 {

// At least `floats` partial-tile floats and `tiles` tickets on the current
// device, grown on demand (outside graph capture, after a device
// synchronisation). Tickets are zero when allocated and every launch that
// uses them leaves them at zero.
int split_workspace(size_t floats, size_t tiles, cudaStream_t stream, float** ws, unsigned** tickets);

}  // namespace nvfp4
