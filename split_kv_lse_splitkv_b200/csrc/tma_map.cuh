// Host-side construction of TMA tensor maps shared by the tensor-core kernels.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace splitkv {

// 3-D bf16 map over a [rows][heads][d] tensor (d contiguous) with a 128-byte-swizzled box
// {64, box_heads, box_rows}: one box is a 64-column half of box_rows x box_heads rows. Returns
// false (with splitkv_last_error() set) if the driver entry point is missing or rejects the map.
bool make_bf16_map(CUtensorMap* map, const void* base, int64_t rows, int heads, int d, int box_heads, int box_rows);

}  // namespace splitkv
