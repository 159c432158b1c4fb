// Host-side TMA tensor maps of the bf16 operands (row-major [rows, 128] views).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hga {

// 2-D tiled map of a [rows, 128] bf16 tensor with boxes of box_rows x 64
// columns and 128-byte swizzle (one box row = one 128-byte swizzle line).
cudaError_t make_bf16_map(CUtensorMap* map, const void* base, int64_t rows, int box_rows);

}  // namespace hga
