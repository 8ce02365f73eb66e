// Host-side TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library needs no link against libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// A row-major byte matrix [rows][row_bytes] seen as 3D (128-byte chunk,
// row, chunk index) with 128-byte swizzle. A box of (128, box_rows,
// box_chunks) lands in shared memory as [chunk][row][128 B] with 16-byte unit
// u of row r stored at unit u ^ (r % 8): threads reading the same unit of 8
// consecutive rows hit 8 different bank groups. Base 16-byte aligned,
// row_bytes a multiple of 128.
bool make_chunked_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows,
                      uint32_t box_chunks);

// A row-major byte matrix [rows][row_bytes] as 2D, box (box_bytes, box_rows),
// box_bytes a multiple of 16. swizzle64 (box_bytes == 64, shared-memory
// destination 512-byte aligned): the 16-byte unit c of box row r lands at
// unit c ^ ((r / 2) % 4), so one 4-byte word per row for 8 consecutive rows
// falls in 8 different banks.
bool make_plain_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_bytes,
                    uint32_t box_rows, bool swizzle64 = false);

// A row-major byte matrix [rows][row_bytes] as 2D, boxes of 32 bytes x
// box_rows rows, 32-byte swizzled: the 16-byte half c of box row r lands at
// half c ^ ((r / 4) % 2), so the same half of 8 consecutive rows falls in 8
// different groups of four banks (shared destination 256-byte aligned).
bool make_rows32_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows);

// Operand tiles for the tensor-core GEMMs: a row-major matrix [rows][K]
// seen in boxes of 128 K-elements x box_rows rows, 128-byte swizzled (rows of
// 128 bytes in shared memory, the K-major layout tcgen05.mma reads).
// u8: one byte per element (E4M3 codes). Base 16-byte aligned, row bytes a
// multiple of 16.
bool make_tile_map_u8(CUtensorMap *map, const void *base, uint64_t rows, uint64_t row_bytes, uint32_t box_rows);
// e2m1: packed E2M1 codes (two per byte, element 2i in the low nibble),
// expanded in shared memory to one byte per element (16 codes in the first 8
// bytes of every 16). Base 32-byte aligned, K a multiple of 128.
bool make_tile_map_e2m1(CUtensorMap *map, const void *base, uint64_t rows, uint64_t K, uint32_t box_rows);

}  // namespace moe
