// Codebook calibration: one round of spherical k-means per subspace
// ("Monodratic: a reproducible sparse attention mixer", section Capacity and
// Figure 3: codebooks calibrated on a training split).  The assignment step
// is the codes kernel with one probe (the codeword of largest score, lower
// index on equal scores); these two kernels do the update:
//
//   calib_partial_kernel   grid (chunks, P): each warp walks a contiguous run
//                          of the chunk's records in order, eight at a time:
//                          turns each record's sub-vector x_s into x_s/|x_s|
//                          (scaled first by the power of two that brings its
//                          largest |coordinate| into [0.5, 1), which is
//                          exact, then multiplied by the correctly rounded
//                          1/sqrt of its sum of squares) and adds it to its
//                          own shared-memory row of the assigned codeword, in
//                          record order; a sub-vector with no nonzero
//                          coordinate is skipped.
//                          The warps' rows are added in warp order and
//                          stored per chunk.
//   calib_finalize_kernel  one CTA per (subspace, codeword): warp w adds
//                          chunks w, w+8, ... in order, the warps' sums are
//                          added in warp order, then normalised; a
//                          codeword with no member, or a zero sum, keeps
//                          the value the round started from.
//
// Every sum has a fixed order, so a round is deterministic.  Records are
// read once per round by each kernel pair (N * D * 4 bytes, plus the
// assignment); the per-chunk sums are P * chunks * K * dsub * 4 bytes, with
// chunks chosen so that this stays below the records' size where possible.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

constexpr int kCalibMaxWarps = 8;
constexpr size_t kCalibSmemBudget = 192 * 1024;

}  // namespace

void calib_plan(long long N, int D, int P, int K, int* chunk, int* nchunk, int* warps) {
  const int dsub = D / P;
  const size_t per_warp = (static_cast<size_t>(K) * dsub + K) * sizeof(float);
  int w = static_cast<int>(kCalibSmemBudget / per_warp);
  w = w < 1 ? 1 : (w > kCalibMaxWarps ? kCalibMaxWarps : w);
  // About two CTAs per SM over all subspaces, at least 16 records per warp,
  // and no more chunks than keep the per-chunk sums (K * dsub floats each)
  // about the size of the records (chunk * dsub floats each).
  const long long target_ctas = 296;
  long long per = (N * P + target_ctas - 1) / target_ctas;
  if (per < 16LL * w) per = 16LL * w;
  const long long max_chunks = N / K + 1;
  long long n = (N + per - 1) / per;
  if (n > max_chunks) { n = max_chunks; per = (N + n - 1) / n; }
  *chunk = static_cast<int>(per);
  *nchunk = static_cast<int>((N + per - 1) / per);
  *warps = w;
}

__global__ void calib_partial_kernel(const CalibArgs a) {
  extern __shared__ float cal_smem[];
  const int dsub = a.D / a.P;
  const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* acc = cal_smem + static_cast<size_t>(warp) * a.K * dsub;
  int* cnt = reinterpret_cast<int*>(cal_smem + static_cast<size_t>(nw) * a.K * dsub) + warp * a.K;
  for (int i = lane; i < a.K * dsub; i += 32) acc[i] = 0.f;
  for (int i = lane; i < a.K; i += 32) cnt[i] = 0;
  __syncwarp();
  grid_dependency_wait();                          // the assignment comes from the codes kernel

  const int s = blockIdx.y;
  const long long r0 = static_cast<long long>(blockIdx.x) * a.chunk;
  const long long r1 = r0 + a.chunk < a.N ? r0 + a.chunk : a.N;
  const long long per = (r1 - r0 + nw - 1) / nw;
  const long long w0 = r0 + warp * per;
  const long long w1 = w0 + per < r1 ? w0 + per : r1;
  const int nj = (dsub + 31) / 32;                 // coordinates per lane (dsub <= 128)
  const float* rec = a.records + s * dsub;
  constexpr int U = 8;                             // records in flight per warp
  for (long long r = w0; r < w1; r += U) {
    float x[U][4], rn[U];
    int code[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long ru = r + u;
      code[u] = ru < w1 ? a.assign[ru * a.P + s] : -1;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = lane + 32 * j;
        x[u][j] = (ru < w1 && j < nj && c < dsub) ? rec[ru * a.D + c] : 0.f;
      }
    }
    // Scale each sub-vector by a power of two (exact) that brings its largest
    // |coordinate| into [0.5, 1), so the sum of squares neither overflows nor
    // underflows; the eight records' sums proceed side by side.
    float ss[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float m = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(x[u][j]));
      const float mx = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
      if (mx == 0.f) code[u] = -1;                 // no direction: not a member
      int ex = 0;
      frexpf(mx, &ex);
      ss[u] = 0.f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[u][j] = ldexpf(x[u][j], -ex);
        ss[u] = __fmaf_rn(x[u][j], x[u][j], ss[u]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < U; ++u) ss[u] += __shfl_xor_sync(0xffffffffu, ss[u], o);
#pragma unroll
    for (int u = 0; u < U; ++u) rn[u] = code[u] >= 0 ? __frsqrt_rn(ss[u]) : 0.f;
    // Add the unit vectors to the codewords' rows in record order.
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (code[u] < 0) continue;
      float* row = acc + code[u] * dsub;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = lane + 32 * j;
        if (j < nj && c < dsub) row[c] += x[u][j] * rn[u];
      }
      if (lane == 0) cnt[code[u]] += 1;
    }
  }
  __syncthreads();
  const long long base = (static_cast<long long>(s) * a.nchunk + blockIdx.x) * a.K;
  for (int i = threadIdx.x; i < a.K * dsub; i += blockDim.x) {
    float v = 0.f;
    for (int w = 0; w < nw; ++w) v += cal_smem[static_cast<size_t>(w) * a.K * dsub + i];
    a.part[base * dsub + i] = v;
  }
  const int* cnts = reinterpret_cast<const int*>(cal_smem + static_cast<size_t>(nw) * a.K * dsub);
  for (int k = threadIdx.x; k < a.K; k += blockDim.x) {
    int c = 0;
    for (int w = 0; w < nw; ++w) c += cnts[w * a.K + k];
    a.pcount[base + k] = c;
  }
}

constexpr int kFinWarps = 8;

__global__ void __launch_bounds__(kFinWarps * 32) calib_finalize_kernel(const CalibArgs a) {
  __shared__ float wsum[kFinWarps][128];
  __shared__ int wcnt[kFinWarps];
  grid_dependency_wait();                          // the sums come from the partial kernel
  const int dsub = a.D / a.P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int s = blockIdx.x / a.K, k = blockIdx.x % a.K;
  // Warp w adds chunks w, w + 8, w + 16, ... in increasing order, eight rows
  // loaded together; the warps' sums are then added in warp order.
  float v[4] = {0.f, 0.f, 0.f, 0.f};
  int cnt = 0;
  constexpr int G = 8;
  for (int c0 = warp; c0 < a.nchunk; c0 += G * kFinWarps) {
    float t[G][4];
    int tc[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int c = c0 + g * kFinWarps;
      const long long row = (static_cast<long long>(s) * a.nchunk + c) * a.K + k;
      tc[g] = c < a.nchunk ? a.pcount[row] : 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int d = lane + 32 * j;
        t[g][j] = (c < a.nchunk && d < dsub) ? a.part[row * dsub + d] : 0.f;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (c0 + g * kFinWarps >= a.nchunk) break;
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] += t[g][j];
      cnt += tc[g];
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int d = lane + 32 * j;
    if (d < dsub) wsum[warp][d] = v[j];
  }
  if (lane == 0) wcnt[warp] = cnt;
  __syncthreads();
  if (warp != 0) return;
  float old[4], ss = 0.f;
  cnt = 0;
  for (int w = 0; w < kFinWarps; ++w) cnt += wcnt[w];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int d = lane + 32 * j;
    v[j] = 0.f;
    if (d < dsub)
      for (int w = 0; w < kFinWarps; ++w) v[j] += wsum[w][d];
    old[j] = d < dsub ? a.cb_old[(static_cast<long long>(s) * a.K + k) * dsub + d] : 0.f;
    ss = __fmaf_rn(v[j], v[j], ss);
  }
  ss = warp_sum(ss);
  const bool keep = cnt == 0 || ss == 0.f;
  const float n = keep ? 1.f : __fsqrt_rn(ss);
  __syncwarp();                                    // every lane has read its old value
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int d = lane + 32 * j;
    if (d < dsub) a.cb_new[(static_cast<long long>(s) * a.K + k) * dsub + d] = keep ? old[j] : __fdiv_rn(v[j], n);
  }
  if (a.counts && lane == 0) a.counts[s * a.K + k] = cnt;
}

cudaError_t launch_calibrate_round(const CalibArgs& a, cudaStream_t st) {
  const int dsub = a.D / a.P;
  const size_t smem = static_cast<size_t>(a.warps) * (static_cast<size_t>(a.K) * dsub + a.K) * sizeof(float);
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(calib_partial_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(calib_partial_kernel, dim3(a.nchunk, a.P), dim3(a.warps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(calib_finalize_kernel, dim3(a.P * a.K), dim3(kFinWarps * 32), 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
