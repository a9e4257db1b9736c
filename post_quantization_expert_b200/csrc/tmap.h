// Host-side creation of TMA tensor maps (the driver's tiled encoder, fetched through the runtime
// so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, box {box_cols, box_rows}, 128-byte
// swizzle, zero fill outside the tensor. Returns cudaErrorInvalidValue if the encoder rejects it.
cudaError_t make_tmap_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, int esize,
                         uint32_t box_rows, uint32_t box_cols);
// 3-D row-major tensor [planes, rows, cols], box {box_cols, box_rows, 1}, 128-byte swizzle.
cudaError_t make_tmap_3d(CUtensorMap* map, const void* base, uint64_t planes, uint64_t rows, uint64_t cols,
                         int esize, uint32_t box_rows, uint32_t box_cols);
