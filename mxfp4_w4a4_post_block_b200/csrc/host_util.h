// Host-side helpers shared by the launchers: driver entry points, device queries.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace batq {

// cuTensorMapEncodeTiled fetched through the runtime (no link-time libcuda dependency,
// so the library loads on machines without a driver).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn();

// 2-D tensor map: dims {inner, outer} in elements, outer stride in bytes, box {bx, by}.
bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                 uint64_t outer_stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// 3-D tensor map (no swizzle): dims {d0, d1, d2} in elements, strides of dims 1 and 2 in bytes.
bool make_map_3d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);

// 3-D tensor map with a swizzle mode (strides need not be increasing).
bool make_map_3d_swizzled(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t d0, uint64_t d1,
                          uint64_t d2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1,
                          uint32_t b2, CUtensorMapSwizzle swizzle);

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace batq
