// Host-side TMA tensor maps (bf16 with 128-byte swizzle unless stated), cached by
// their parameters so that a repeated call re-encodes nothing.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace mla {

// 2-D map over `rows` rows of `cols` bf16 values, rows `row_bytes` apart; boxes of
// box_rows x box_cols (box_cols * 2 <= 128).
bool tma_map_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                uint32_t box_cols, uint32_t box_rows);

// 3-D map: dims (d0 values, d1, d2) with byte strides s1 (dim 1) and s2 (dim 2);
// boxes of b2 x b1 x b0.
bool tma_map_3d(CUtensorMap* m, const void* ptr, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2);

// Map of rank 1..5: dims[i] values along dimension i (dimension 0 contiguous),
// strides[i] the byte stride of dimension i + 1 (any order, multiples of 16),
// boxes of box[i] values.  The box lands in shared memory with dimension 0
// fastest, so a stride smaller than the row pitch can order several chunks of a
// row one after another.  `bytes`: 1-byte elements (e4m3 codes) instead of bf16;
// swizzle_bytes: 128, 64, 32 or 0 (none).
bool tma_map_nd(CUtensorMap* m, const void* ptr, uint32_t rank, const uint64_t* dims, const uint64_t* strides,
                const uint32_t* box, bool bytes = false, int swizzle_bytes = 128);

}  // namespace mla
