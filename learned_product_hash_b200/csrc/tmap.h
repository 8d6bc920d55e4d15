// TMA tensor maps over the token-major [rows, H, D] bf16 tensors of the
// library (q, k, v, their rotated copies, gradients): viewed as a 3-D tensor
// (D, H, rows) with a (64, 1, BS) box and 128-byte swizzle, so one box is
// 64 coordinates of one head for BS consecutive tokens -- one 128-byte row per
// token, the layout the tensor-core operand descriptors expect.
#pragma once

#include <cuda.h>

namespace mdr {

// False when the driver entry point is missing or the encoder rejects the
// map (base not 16-byte aligned, strides not multiples of 16 bytes, ...).
bool make_tile_map(CUtensorMap* m, const void* ptr, long long rows, int H, int D, int BS);

}  // namespace mdr
