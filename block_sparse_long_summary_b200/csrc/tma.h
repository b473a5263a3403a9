// Host-side TMA tensor-map encoding (2-D, bf16, 128-byte swizzle) through the driver entry
// point, so the library needs no link-time dependency on libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace cobs {

// Encode a 2-D row-major bf16 tensor [rows, cols] (cols contiguous) read in boxes of
// box_rows x 64 columns (128 bytes, 128-byte swizzle). Returns false on failure.
bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);

// 3-D bf16 tensor (dims[0] contiguous; strides in bytes of dims 1 and 2) read in boxes of
// 64 x box[1] x box[2] elements with 128-byte swizzle.
bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                         const uint32_t box[3]);

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace cobs
