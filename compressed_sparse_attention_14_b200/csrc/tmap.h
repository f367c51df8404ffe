// Host-side TMA tensor-map encoding for libcsa. cuTensorMapEncodeTiled is
// reached through the runtime's driver entry point, so the library does not
// link libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa {

// Row-major bf16 matrix [rows, cols] (cols contiguous, row pitch `pitch_elems`)
// viewed as 2D tiles of box_rows x box_cols (box_cols * 2 <= 128 bytes) with
// 128-byte swizzle. Returns false if the driver rejects the map.
bool make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_elems,
                       uint32_t box_rows, uint32_t box_cols);

// The same for a byte matrix (e4m3 values): row pitch in bytes, box_cols <= 128.
bool make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                     uint32_t box_rows, uint32_t box_cols);

// Rows of a bf16 matrix that come in blocks: rows_per_block rows of `cols`
// elements (row pitch cols, 16-byte multiple), block j at j * block_bytes;
// viewed as 3D tiles of box_blocks x rows_per_block x box_cols with 128-byte
// swizzle (the tile lands in shared memory exactly as box_blocks *
// rows_per_block consecutive rows of a 2D tile would).
bool make_tmap_bf16_blocks(CUtensorMap* map, const void* base, uint64_t nblocks, uint32_t rows_per_block,
                           uint64_t cols, uint64_t block_bytes, uint32_t box_blocks, uint32_t box_cols);

}  // namespace csa
