// Host-side TMA tensor-map encoding.  The driver entry point is fetched
// through the runtime (cudaGetDriverEntryPoint), so the library does not
// link libcuda directly and can be loaded on a machine without a driver.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace dash {

// Encode a 3-D tiled map over fp16 data laid out as depth x rows x cols
// (cols innermost, cols a multiple of 64): box {64, box_rows, 1}, 128-byte
// swizzle.  Returns cudaSuccess or cudaErrorInvalidValue.
cudaError_t encode_f16_3d_map(CUtensorMap* map, const void* base, int cols, int rows, long long depth,
                              int box_rows);

// Encode a 3-D tiled map over a split stack: dims {B (columns, innermost),
// B (rows), 2 * nmat (matrix * 2 + plane)} of fp16, box {64, box_rows, 1},
// 128-byte swizzle.  Returns cudaSuccess or cudaErrorInvalidValue.
cudaError_t encode_split_stack_map(CUtensorMap* map, const void* base, int B, int nmat, int box_rows = 128);

// Encode a 3-D tiled map for 32 x 32 epilogue steps of a stack of B x B
// matrices: split fp16 (f32 = false: dims {B, B, depth = 2 * nmat}, box
// {32, 32, 2}, both planes, 64-byte swizzle) or fp32 (dims {B, B, depth =
// nmat}, box {32, 32, 1}, 128-byte swizzle).  base must be 16-byte aligned.
// Returns cudaSuccess or cudaErrorInvalidValue.
cudaError_t encode_epilogue_map(CUtensorMap* map, void* base, bool f32, int B, long long depth);

}  // namespace dash
