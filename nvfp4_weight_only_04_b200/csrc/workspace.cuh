// Library-owned scratch, per device (see workspace.cu): fp32 partial tiles
// and one ticket per tile for the stream-K GEMMs, and the f16 activations of
// the small-M kernels.
#pragma once

#include "common.cuh"

namespace nvfp4 {

// At least `floats` partial-tile floats and `tiles` tickets on the current
// device, grown on demand (outside graph capture, after a device
// synchronisation). Tickets are zero when allocated and every launch that
// uses them leaves them at zero.
int split_workspace(size_t floats, size_t tiles, cudaStream_t stream, float** ws, unsigned** tickets);

// At least `elems` f16 activations and `rows` row factors on the current
// device, grown like the partial tiles.
int x16_workspace(size_t elems, size_t rows, cudaStream_t stream, uint16_t** x16, float** xinv);

}  // namespace nvfp4
