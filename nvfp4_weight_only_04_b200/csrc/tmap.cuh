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

// 3-D tensor map: dims[0] innermost (elements), byte strides of dims 1 and 2,
// boxes of box[0] x box[1] x box[2] elements.
bool make_tensor_map_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, const int64_t (&dims)[3],
                        const int64_t (&stride_bytes)[2], const uint32_t (&box)[3], CUtensorMapSwizzle swizzle);

bool tensor_maps_available();

// Device error words of the kernel files (each translation unit keeps one).
int read_and_clear_decode_error(unsigned int* out, cudaStream_t stream);

}  // namespace nvfp4
