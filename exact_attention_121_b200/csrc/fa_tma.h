// Host helpers for TMA tensor maps over (batch, seqlen, heads, headdim)
// tensors: the driver's cuTensorMapEncodeTiled is reached through the runtime's
// driver entry point, so the library needs no link against libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

// True when the driver exposes the tensor-map encoder.
bool tma_available();

// 4-D map (D, H, S, B) of 16-bit elements with a box of 64 head-dim elements x
// 1 head x `box_rows` rows x 1 batch, 128-byte swizzle, zero fill outside the
// tensor.  Returns false if the encoder is missing or rejects the map.
bool make_bshd_map(CUtensorMap* m, const void* base, bool bf16, int D, int H, int S, int B, int box_rows);
// Same with element strides (batch, token, head) of a tensor whose head
// dimension is contiguous; every stride must be a multiple of 8 elements.
bool make_bshd_map_strided(CUtensorMap* m, const void* base, bool bf16, int D, int H, int S, int B,
                           const long long st[3], int box_rows);

// 4-D map (D, H, S, B) of packed 8-bit elements (E4M3 codes) with a box of
// all D head-dim elements (D bytes) x 1 head x `box_rows` rows x 1 batch,
// 128-byte swizzle (D = 128) or 64-byte swizzle (D = 64), zero fill outside
// the tensor.
bool make_bshd_map_u8(CUtensorMap* m, const void* base, int D, int H, int S, int B, int box_rows);

// 4-D map (D, H, S, B) of fp32 elements with a box of all D elements x 1 head
// x `box_rows` rows x 1 batch, no swizzle (dense row-major box in shared
// memory); used as the target of tiled reductions.
bool make_bshd_map_f32(CUtensorMap* m, const void* base, int D, int H, int S, int B, int box_rows);

}  // namespace fa
