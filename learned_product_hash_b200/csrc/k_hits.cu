// Target-block hit diagnostic: for every route with a target block, whether
// the target is among the route's selected blocks (remote or local part),
// and the number of routes with a target and of hits.  "Monodratic: a
// reproducible sparse attention mixer", section Evidence (the target-block
// hit rate of the associative-recall run).
//
// One CTA of 1024 threads strides over the routes (a route reads its R + L
// selected ids and its target: a few bytes each, so even the 128K workload's
// 32K routes are a few microseconds); the counts are reduced in a fixed
// order (warp shuffles, then the warps' partials in warp order), so the
// result needs no zeroing and no atomics.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

constexpr int kHitsThreads = 1024;

__global__ void __launch_bounds__(kHitsThreads) hits_kernel(const HitsArgs a) {
  __shared__ int part[kHitsThreads / 32][2];
  grid_dependency_wait();
  int nt = 0, nh = 0;
  for (long long r = threadIdx.x; r < a.nroutes; r += kHitsThreads) {
    const int t = a.target[r];
    int h = -1;
    if (t >= 0) {
      const int32_t* row = a.sel + r * a.nsel;
      h = 0;
      for (int i = 0; i < a.nsel; ++i) h |= row[i] == t ? 1 : 0;
      ++nt;
      nh += h;
    }
    if (a.hit) a.hit[r] = h;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    nt += __shfl_xor_sync(0xffffffffu, nt, o);
    nh += __shfl_xor_sync(0xffffffffu, nh, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { part[warp][0] = nt; part[warp][1] = nh; }
  __syncthreads();
  if (threadIdx.x == 0) {
    int st = 0, sh = 0;
    for (int w = 0; w < kHitsThreads / 32; ++w) { st += part[w][0]; sh += part[w][1]; }
    a.counts[0] = st;
    a.counts[1] = sh;
  }
}

cudaError_t launch_hits(const HitsArgs& a, cudaStream_t st) {
  cudaError_t e = launch_pdl(hits_kernel, dim3(1), dim3(kHitsThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
