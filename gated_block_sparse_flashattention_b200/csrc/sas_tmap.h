// Host helper: TMA tensor maps for [outer, rows, inner] bf16 tensors with a
// 128-byte swizzle (the layout the tcgen05 shared-memory descriptors expect).
#pragma once

#include <cstdint>
#include <cuda.h>

namespace sas {

// Encodes a 3-D map over a contiguous bf16 tensor [outer][rows][inner] with box
// (64 elements, box_rows, 1). Out-of-range rows read as zero. Returns false if
// the driver entry point is unavailable or the encode call fails.
bool make_tmap_bf16_3d(CUtensorMap* out, const void* base, uint64_t inner, uint64_t rows, uint64_t outer,
                       uint32_t box_rows);

// Encodes a 2-D map over a contiguous bf16 matrix [rows][inner] (inner <= 256)
// with box (inner, box_rows) and no swizzle: a box lands as box_rows dense rows.
bool make_tmap_bf16_rows(CUtensorMap* out, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);

}  // namespace sas
