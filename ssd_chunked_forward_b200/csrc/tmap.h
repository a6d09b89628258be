// tmap.h -- host-side creation of TMA tensor maps (driver entry point fetched
// at run time through the CUDA runtime, so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// A 4-D bf16 tensor map over a row-major [d3][d2][d1][d0] array (d0
// innermost; for the token tensors d3 = batch, d2 = tokens, d1 = heads or
// groups), box (64, 1, rows, 1) with 128-byte swizzle: one box is `rows`
// tokens of 64 elements = 128 bytes, landing in shared memory as rows of 128
// bytes.  Rows past d2 read as zero and are not stored, so a box never
// crosses into the next batch row.  Returns cudaSuccess or an error (bad
// alignment, missing driver entry point).
cudaError_t make_tmap_bf16_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint64_t d3, uint32_t box_rows);

// A 4-D fp32 tensor map over a row-major [d3][d2][d1][d0] array (d0 <= 256
// innermost, e.g. the per-state log-decays [B][T][H][N]), box (d0, 1, rows,
// 1) without swizzle: one box lands as `rows` dense rows of d0 floats.  Rows
// past d2 read as zero.
cudaError_t make_tmap_f32_4d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                             uint64_t d3, uint32_t box_rows);

// A 2-D fp32 tensor map over a row-major [rows][64] array, box (32, 128) with
// 128-byte swizzle: one box is 128 rows of 32 floats = 128 bytes; a 128 x 64
// tile is two boxes (columns 0-31 and 32-63).
cudaError_t make_tmap_f32_rows64(CUtensorMap* map, const void* base, uint64_t rows);

}  // namespace ssd
