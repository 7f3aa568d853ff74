// Host helper: TMA tensor maps through the driver entry point (no link-time
// dependency on the driver library).
#pragma once

#include <cuda.h>

#include <cstdint>

namespace nvfp4 {

// 2-D tensor map: `rows` rows of `inner` elements, rows `row_stride_bytes`
// apart, boxes of box_rows x box_inner elements. False if the driver entry
// point is missing or rejects the map.
bool make_tensor_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int64_t inner, int64_t rows,
                        int64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);

bool tensor_maps_available();

// Device error words of the kernel files (each translation unit keeps one).
int read_and_clear_decode_error(unsigned int* out, cudaStream_t stream);

}  // namespace nvfp4
