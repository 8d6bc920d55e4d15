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
// float32 partial sums (dimensions d mod 4) added pairwise at the end (the
// kernel is instantiated per dsub so that the loop unrolls completely).  The
// selected codewords are taken by rounds of warp arg-max, best first: the
// highest score by one warp max-reduction of an order-preserving integer
// image of the score, then the lowest index among the lanes holding it (a NaN
// score counts as -inf).

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

constexpr int kCodeWarps = 16;
constexpr int kMaxK = 128;

// Order-preserving map of a float32 (not NaN) to uint32.
__device__ __forceinline__ uint32_t ordered_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace

template <int F4>   // dsub / 4
__global__ void __launch_bounds__(kCodeWarps * 32)
codes_kernel(const __grid_constant__ CodesArgs a) {
  extern __shared__ float4 csm4[];
  constexpr int dsub = 4 * F4, RS = dsub + 4;                 // codebook row stride (floats)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = a.D;
  float* cbs = reinterpret_cast<float*>(csm4);                // [P][K][dsub + 4]
  float* xs = cbs + a.P * a.K * RS + warp * D;                // this warp's summary row

  // The codebooks are staged before waiting on the previous kernel (they are
  // an input of the forward), unless the previous kernel writes them.
  if (a.codebooks_written_before) grid_dependency_wait();
  for (int i4 = threadIdx.x; i4 < a.K * D / 4; i4 += kCodeWarps * 32) {
    const int i = 4 * i4, row = i / dsub, d = i - row * dsub;  // row = sdx * K + k
    *reinterpret_cast<float4*>(cbs + row * RS + d) = reinterpret_cast<const float4*>(a.codebooks)[i4];
  }
  __syncthreads();
  if (!a.codebooks_written_before) grid_dependency_wait();   // the summaries come from the previous kernel

  const int nbr = a.nbr > 0 ? a.nbr : a.nb;         // blocks a.j0 .. a.j0 + nbr - 1
  const long long rows0 = a.xbar[0] ? static_cast<long long>(a.B) * a.H[0] * nbr : 0;
  const long long rows1 = a.xbar[1] ? static_cast<long long>(a.B) * a.H[1] * nbr : 0;
  const long long nwarps = static_cast<long long>(gridDim.x) * kCodeWarps;
  for (long long row = static_cast<long long>(blockIdx.x) * kCodeWarps + warp; row < rows0 + rows1; row += nwarps) {
    const int side = row < rows0 ? 0 : 1;
    const long long rl = side ? row - rows0 : row;
    const long long rr = (rl / nbr) * a.nb + a.j0 + rl % nbr;  // (b * H + h) * nb + j
    const float* xb = a.xbar[side] + rr * D;
    for (int d4 = lane; d4 < D / 4; d4 += 32)
      reinterpret_cast<float4*>(xs)[d4] = __ldg(reinterpret_cast<const float4*>(xb) + d4);
    __syncwarp();
    const int need = side == 0 ? a.probes : 1;
    int addr = 0;
    for (int sdx = 0; sdx < a.P; ++sdx) {
      const float4* xs4 = reinterpret_cast<const float4*>(xs + sdx * dsub);
      uint32_t key[kMaxK / 32];        // ordered score; 0 = no codeword (no float maps to 0)
#pragma unroll
      for (int m = 0; m < kMaxK / 32; ++m) {
        const int k = lane + 32 * m;
        key[m] = 0;
        if (k < a.K) {
          const float4* cw = reinterpret_cast<const float4*>(cbs + (sdx * a.K + k) * RS);
          float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
#pragma unroll
          for (int d4 = 0; d4 < F4; ++d4) {
            const float4 xv = xs4[d4], cv = cw[d4];
            acc0 = __fmaf_rn(xv.x, cv.x, acc0);
            acc1 = __fmaf_rn(xv.y, cv.y, acc1);
            acc2 = __fmaf_rn(xv.z, cv.z, acc2);
            acc3 = __fmaf_rn(xv.w, cv.w, acc3);
          }
          const float v = __fadd_rn(__fadd_rn(acc0, acc1), __fadd_rn(acc2, acc3));
          key[m] = ordered_bits(v == v ? v : -INFINITY);
        }
      }
      for (int rnd = 0; rnd < need; ++rnd) {
        // This lane's best: highest key, lowest index (m ascending).
        uint32_t lk = key[0];
        int lm = 0;
#pragma unroll
        for (int m = 1; m < kMaxK / 32; ++m)
          if (key[m] > lk) { lk = key[m]; lm = m; }
        const uint32_t top = __reduce_max_sync(0xffffffffu, lk);
        const int bi = static_cast<int>(
            __reduce_min_sync(0xffffffffu, lk == top ? static_cast<uint32_t>(lane + 32 * lm) : 0xffffffffu));
        if (side == 0) {
          if (lane == 0) a.qcodes[(rr * a.P + sdx) * a.probes + rnd] = bi;
#pragma unroll
          for (int m = 0; m < kMaxK / 32; ++m)
            if (lane + 32 * m == bi) key[m] = 0;
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
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return cudaErrorInvalidValue;
  const long long rows = (a.xbar[0] ? static_cast<long long>(a.B) * a.H[0] * nbr : 0) +
                         (a.xbar[1] ? static_cast<long long>(a.B) * a.H[1] * nbr : 0);
  if (rows == 0) return cudaSuccess;
  if (a.K > kMaxK || a.P > 4) return cudaErrorInvalidValue;
  const size_t smem =
      (static_cast<size_t>(a.P) * a.K * (a.D / a.P + 4) + static_cast<size_t>(kCodeWarps) * a.D) * sizeof(float);
  void (*k)(CodesArgs) = nullptr;
  switch (a.D / a.P / 4) {
    case 2: k = codes_kernel<2>; break;
    case 4: k = codes_kernel<4>; break;
    case 8: k = codes_kernel<8>; break;
    case 16: k = codes_kernel<16>; break;
    case 32: k = codes_kernel<32>; break;
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sms = cached_sm_count();
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(k), kCodeWarps * 32, smem);
  if (sms <= 0) return cudaErrorUnknown;
  if (per_sm < 1) per_sm = 1;
  const long long need = (rows + kCodeWarps - 1) / kCodeWarps;
  const long long cap = static_cast<long long>(sms) * (per_sm < 2 ? per_sm : 2);
  const unsigned grid = static_cast<unsigned>(need < cap ? need : cap);
  e = launch_pdl(k, dim3(grid), dim3(kCodeWarps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
