// K2: product codes of the block summaries.
//
//   keys    : per subspace the codeword of largest <kbar_s, C[s,k]> (lowest
//             index on equal scores) -> product address sum_s c_s K^(P-1-s);
//   queries : per subspace the p codewords of largest score, best first.
// Pages: "Monodratic Claims Learned Routing Can Make Sparse Causal Attention
// More Selective", section "Monodratic Turns Sparse Attention Into a
// Retrieval Decision" (a block's address is a combination of several code
// choices; a query probes the best few codes of each subspace), and
// "Monodratic: a reproducible sparse attention mixer", section Mixer.
//
// One warp per summary row (side, b, h, j), 16 warps per CTA, about two CTAs
// per SM so that the rows' memory latency overlaps.  Each CTA first copies the
// codebooks into shared memory, one row per codeword padded to dsub + 4
// words, so that the 16-byte reads of 32 lanes -- one codeword each -- spread
// over all banks.  A lane scores its codewords over the subspace with four
// float32 partial sums (dimensions d mod 4) added pairwise at the end; the
// selected codewords are then taken by rounds of warp arg-max (higher score,
// lower index on equal scores; a NaN score counts as -inf), best first.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

constexpr int kCodeWarps = 16;
constexpr int kMaxK = 128;

}  // namespace

__global__ void __launch_bounds__(kCodeWarps * 32)
codes_kernel(const __grid_constant__ CodesArgs a) {
  extern __shared__ float4 csm4[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.D, dsub = D / a.P, RS = dsub + 4;           // codebook row stride (floats)
  float* cbs = reinterpret_cast<float*>(csm4);                // [P][K][dsub + 4]
  float* xs = cbs + a.P * a.K * RS + warp * D;                // this warp's summary row

  for (int i = threadIdx.x; i < a.K * D; i += kCodeWarps * 32) {
    const int row = i / dsub, d = i - row * dsub;              // row = sdx * K + k
    cbs[row * RS + d] = __ldg(a.codebooks + i);
  }
  __syncthreads();
  grid_dependency_wait();          // the summaries come from the previous kernel

  const long long rows0 = a.xbar[0] ? static_cast<long long>(a.B) * a.H[0] * a.nb : 0;
  const long long rows1 = a.xbar[1] ? static_cast<long long>(a.B) * a.H[1] * a.nb : 0;
  const long long nwarps = static_cast<long long>(gridDim.x) * kCodeWarps;
  for (long long row = static_cast<long long>(blockIdx.x) * kCodeWarps + warp; row < rows0 + rows1; row += nwarps) {
    const int side = row < rows0 ? 0 : 1;
    const long long rr = side ? row - rows0 : row;             // (b * H + h) * nb + j
    const float* xb = a.xbar[side] + rr * D;
    for (int d4 = lane; d4 < D / 4; d4 += 32)
      reinterpret_cast<float4*>(xs)[d4] = __ldg(reinterpret_cast<const float4*>(xb) + d4);
    __syncwarp();
    const int need = side == 0 ? a.probes : 1;
    int addr = 0;
    for (int sdx = 0; sdx < a.P; ++sdx) {
      const float4* xs4 = reinterpret_cast<const float4*>(xs + sdx * dsub);
      float sc[kMaxK / 32];
      int ki[kMaxK / 32];
#pragma unroll
      for (int m = 0; m < kMaxK / 32; ++m) {
        const int k = lane + 32 * m;
        sc[m] = -INFINITY;
        ki[m] = 0x7fffffff;
        if (k < a.K) {
          const float4* cw = reinterpret_cast<const float4*>(cbs + (sdx * a.K + k) * RS);
          float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 4
          for (int d4 = 0; d4 < dsub / 4; ++d4) {
            const float4 xv = xs4[d4], cv = cw[d4];
            acc0 = __fmaf_rn(xv.x, cv.x, acc0);
            acc1 = __fmaf_rn(xv.y, cv.y, acc1);
            acc2 = __fmaf_rn(xv.z, cv.z, acc2);
            acc3 = __fmaf_rn(xv.w, cv.w, acc3);
          }
          const float v = __fadd_rn(__fadd_rn(acc0, acc1), __fadd_rn(acc2, acc3));
          sc[m] = v == v ? v : -INFINITY;
          ki[m] = k;
        }
      }
      for (int rnd = 0; rnd < need; ++rnd) {
        float bsc = sc[0];
        int bi = ki[0];
#pragma unroll
        for (int m = 1; m < kMaxK / 32; ++m)
          if (better(sc[m], ki[m], bsc, bi)) { bsc = sc[m]; bi = ki[m]; }
        warp_best(bsc, bi);
        if (side == 0) {
          if (lane == 0) a.qcodes[(rr * a.P + sdx) * a.probes + rnd] = bi;
#pragma unroll
          for (int m = 0; m < kMaxK / 32; ++m)
            if (ki[m] == bi) { sc[m] = -INFINITY; ki[m] = 0x7fffffff; }
        } else {
          addr = addr * a.K + bi;
        }
      }
    }
    if (side == 1 && lane == 0) a.addr[rr] = addr;
    __syncwarp();
  }
}

cudaError_t launch_codes(const CodesArgs& a, cudaStream_t st) {
  const long long rows = (a.xbar[0] ? static_cast<long long>(a.B) * a.H[0] * a.nb : 0) +
                         (a.xbar[1] ? static_cast<long long>(a.B) * a.H[1] * a.nb : 0);
  if (rows == 0) return cudaSuccess;
  if (a.K > kMaxK || a.P > 4) return cudaErrorInvalidValue;
  const size_t smem =
      (static_cast<size_t>(a.P) * a.K * (a.D / a.P + 4) + static_cast<size_t>(kCodeWarps) * a.D) * sizeof(float);
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(codes_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sms = cached_sm_count();
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(codes_kernel), kCodeWarps * 32, smem);
  if (sms <= 0) return cudaErrorUnknown;
  if (per_sm < 1) per_sm = 1;
  const long long need = (rows + kCodeWarps - 1) / kCodeWarps;
  const long long cap = static_cast<long long>(sms) * (per_sm < 2 ? per_sm : 2);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  e = launch_pdl(codes_kernel, dim3(grid), dim3(kCodeWarps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
