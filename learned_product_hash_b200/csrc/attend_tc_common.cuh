// Device helpers shared by the two tensor-core attention kernels (one query
// head per tile, and one pair of query heads of a KV-head group per unit).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "tc_ptx.cuh"

namespace mdr {
namespace atc {

// Wall-time bound of every mbarrier wait in the attention kernels.
constexpr uint64_t kWaitNs = 2000000000ull;

// Valid entries of a sel row are ids in [0, j]; everything else is skipped.
__device__ __forceinline__ bool valid_id(int id, int j) { return id >= 0 && id <= j; }

// Wait for the phase with the given parity; give up after kWaitNs of wall
// time or once another role has set the abort flag.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  using namespace tc;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitNs) return false;
  }
}

// 2^x on the special-function unit (ex2.approx.ftz: about 2 ulp, subnormal
// results flush to zero, which the softmax weights tolerate).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats rounded to bf16, a in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

}  // namespace atc
}  // namespace mdr
