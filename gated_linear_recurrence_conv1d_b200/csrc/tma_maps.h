// tma_maps.h -- host-side construction of the TMA tensor maps the tensor-core kernels use
// (cuTensorMapEncodeTiled reached through the runtime's driver entry point).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace rglru {
namespace tc {

// 3-D map of a bf16 [B][T][W] tensor (W contiguous): box box_c channels x box_t tokens x 1 row,
// no swizzle, out-of-range elements read as zero (a load may start at a negative token).
bool make_map_3d(CUtensorMap* m, const void* base, int W, int T, int B, int box_c, int box_t);

// 3-D map of a bf16 [D2][D1][W] tensor (W contiguous) whose box rows are box_c = 64 channels
// (128 bytes), loaded and stored in the 128-byte swizzle; box box_c x box_r x 1.
bool make_map_3d_sw128(CUtensorMap* m, const void* base, int W, int D1, int D2, int box_c, int box_r);

// 3-D map of a bf16 [d2][d1][d0] tensor (d0 contiguous) with any box b0 x b1 x b2, b0 = 64
// elements (128 bytes), in the 128-byte swizzle.
bool make_map_3d_box_sw128(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t b0,
                           uint32_t b1, uint32_t b2);

// 2-D map (inner x outer elements of bf16 or fp32, rows row_bytes apart) whose box rows are
// exactly 128 bytes, loaded and stored in the 128-byte swizzle.
bool make_map_2d_sw128_elem(CUtensorMap* m, const void* base, uint32_t elem_bytes, uint64_t inner, uint64_t outer,
                            uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);
bool make_map_2d_sw128(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                       uint32_t box_inner, uint32_t box_outer);

}  // namespace tc
}  // namespace rglru
