// tmap.h -- host-side creation of TMA tensor maps (driver entry point fetched
// at run time through the CUDA runtime, so the library does not link libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

// A 3-D bf16 tensor map over a row-major [d2][d1][d0] array (d0 innermost),
// box (64, 1, rows) with 128-byte swizzle: one box is `rows` rows of 64
// elements = 128 bytes, landing in shared memory as rows of 128 bytes.
// Returns cudaSuccess or an error (bad alignment, missing driver entry point).
cudaError_t make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint32_t box_rows);

// A 2-D fp32 tensor map over a row-major [rows][64] array, box (32, 128) with
// 128-byte swizzle: one box is 128 rows of 32 floats = 128 bytes; a 128 x 64
// tile is two boxes (columns 0-31 and 32-63).
cudaError_t make_tmap_f32_rows64(CUtensorMap* map, const void* base, uint64_t rows);

}  // namespace ssd
