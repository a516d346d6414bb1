// Tensor maps for TMA tile loads of bf16 K-major operands (host side).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace moe {

constexpr int kTmapBoxK = 64;  // K elements per box: one 128-byte swizzle row of bf16

// [rows, K] row-major bf16, box = 64 (K) x box_rows, 128-byte swizzle; reads
// past either edge return zeros.  False if the driver rejects the map (base
// not 16-byte aligned, K * 2 not a multiple of 16, ...).
bool make_tmap_bf16_2d(CUtensorMap *m, const void *base, int64_t rows, int K, int box_rows);

// [E, Nw, K] bf16, box = 64 (K) x box_rows x 1, 128-byte swizzle, zero fill.
bool make_tmap_bf16_3d(CUtensorMap *m, const void *base, int E, int Nw, int K, int box_rows);

// [rows, cols] row-major fp32, box = box_cols x box_rows, no swizzle, zero
// fill past either edge (cols * 4 must be a multiple of 16).
bool make_tmap_f32_2d(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows, int box_cols);

}  // namespace moe
