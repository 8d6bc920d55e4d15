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
// codebooks into shared memory transposed to [subspace][dimension][codeword],
// so that the lanes of a warp -- one codeword each -- read consecutive words.
// A lane scores its codewords over the subspace with four float32 partial
// sums (dimensions d mod 4) added pairwise at the end; the rank of a codeword
// is the number of codewords with a higher score or an equal score and a
// lower index, so ranks 0 .. need-1 are the selected codewords in order (a
// NaN score counts as -inf).

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

constexpr int kCodeWarps = 16;
constexpr int kMaxK = 128;

}  // namespace

__global__ void __launch_bounds__(kCodeWarps * 32)
codes_kernel(const __grid_constant__ CodesArgs a) {
  extern __shared__ float csm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.D, dsub = D / a.P;
  float* cbt = csm;                                           // [P][dsub][K]
  float* wsm = csm + a.K * D + warp * (D + kMaxK + 4);        // this warp: mean [D], scores [K], best [4]
  float* xs = wsm;
  float* scs = wsm + D;
  int* best = reinterpret_cast<int*>(wsm + D + kMaxK);

  for (int i = threadIdx.x; i < a.K * D; i += kCodeWarps * 32) {
    const int sdx = i / (a.K * dsub), r = i % (a.K * dsub), k = r / dsub, d = r % dsub;
    cbt[(sdx * dsub + d) * a.K + k] = __ldg(a.codebooks + i);
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
    for (int sdx = 0; sdx < a.P; ++sdx) {
      const float4* xs4 = reinterpret_cast<const float4*>(xs + sdx * dsub);
      const float* cw = cbt + sdx * dsub * a.K;
      for (int k = lane; k < a.K; k += 32) {
        float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll 4
        for (int d4 = 0; d4 < dsub / 4; ++d4) {
          const float4 xv = xs4[d4];
          const float* c4 = cw + 4 * d4 * a.K + k;
          acc0 = __fmaf_rn(xv.x, c4[0], acc0);
          acc1 = __fmaf_rn(xv.y, c4[a.K], acc1);
          acc2 = __fmaf_rn(xv.z, c4[2 * a.K], acc2);
          acc3 = __fmaf_rn(xv.w, c4[3 * a.K], acc3);
        }
        const float sc = __fadd_rn(__fadd_rn(acc0, acc1), __fadd_rn(acc2, acc3));
        scs[k] = sc == sc ? sc : -INFINITY;
      }
      __syncwarp();
      for (int k = lane; k < a.K; k += 32) {
        const float sc = scs[k];
        int rank = 0;
#pragma unroll 4
        for (int k2 = 0; k2 < a.K; ++k2) {
          const float s2 = scs[k2];
          rank += (s2 > sc || (s2 == sc && k2 < k)) ? 1 : 0;
        }
        if (rank < need) {
          if (side == 0)
            a.qcodes[(rr * a.P + sdx) * a.probes + rank] = k;
          else
            best[sdx] = k;
        }
      }
      __syncwarp();
    }
    if (side == 1 && lane == 0) {
      int addr = 0;
      for (int sdx = 0; sdx < a.P; ++sdx) addr = addr * a.K + best[sdx];
      a.addr[rr] = addr;
    }
    __syncwarp();
  }
}

cudaError_t launch_codes(const CodesArgs& a, cudaStream_t st) {
  const long long rows = (a.xbar[0] ? static_cast<long long>(a.B) * a.H[0] * a.nb : 0) +
                         (a.xbar[1] ? static_cast<long long>(a.B) * a.H[1] * a.nb : 0);
  if (rows == 0) return cudaSuccess;
  if (a.K > kMaxK || a.P > 4) return cudaErrorInvalidValue;
  const size_t smem = (static_cast<size_t>(a.K) * a.D + static_cast<size_t>(kCodeWarps) * (a.D + kMaxK + 4)) *
                      sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(codes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, codes_kernel, kCodeWarps * 32, smem)) !=
      cudaSuccess)
    return e;
  if (per_sm < 1) per_sm = 1;
  const long long need = (rows + kCodeWarps - 1) / kCodeWarps;
  const long long cap = static_cast<long long>(sms) * (per_sm < 2 ? per_sm : 2);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  e = launch_pdl(codes_kernel, dim3(grid), dim3(kCodeWarps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
