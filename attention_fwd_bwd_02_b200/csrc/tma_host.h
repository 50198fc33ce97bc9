// tma_host.h -- host-side construction of TMA tensor maps for the bf16 /
// fp16 operands (Q, K, V, dO, ...).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa_common.cuh"

namespace fa {

// Tensor map over a bf16 (p.f16 = 0), fp16 (p.f16 = 1) or e4m3 (p.f8 = 1)
// operand with S rows per head, read as boxes of 128-byte rows (64 16-bit or
// 128 8-bit columns) x box_rows rows with 128-byte swizzle (the canonical K-major /
// MN-major operand layout of tcgen05).  Coordinates (x, row, z):
//   BNSD: x = column 0..D-1, z = b*N + h;   BSH: x = h*D + column, z = b.
// Rows past S read as zeros.
cudaError_t make_operand_map(CUtensorMap* map, const void* base,
                             const Problem& p, int S, int box_rows);

// Tensor map over an fp32 [planes][rows][cols] array (cols contiguous),
// boxes of box_cols x box_rows, no swizzle.  Used for the tiled reduce-add
// into the dQ accumulator; elements outside the array are skipped.
cudaError_t make_f32_rows_map(CUtensorMap* map, const void* base, int cols,
                              int rows, int64_t planes, int box_cols,
                              int box_rows);

}  // namespace fa
