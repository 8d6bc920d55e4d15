// K4: probe -> fixed candidate slots -> rerank -> top-R, plus L local blocks.
//
// One warp per route (sequence b, query head hq, query block j).  The probed
// addresses are the product of the p best codewords of each subspace (first
// subspace's rank slowest).  Each probed address owns cap candidate slots:
// the stored blocks of its list that are remote-eligible, i <= j - L; lists
// hold ascending ids, so those are a prefix and the walk stops at the first
// later block.  Candidates are scored by <qbar_j, kbar_i> in float32 (lanes
// split the head dimension, a butterfly sum combines them), the R best are
// kept (higher score first, lower id on equal scores) and written in
// ascending id order, -1 padded; then the local blocks j-L+1..j.
// Pages: "Monodratic Claims Learned Routing Can Make Sparse Causal Attention
// More Selective", section "Monodratic Turns Sparse Attention Into a
// Retrieval Decision" (probe, candidates, rerank, fixed number of remote
// blocks, guaranteed local blocks); "Monodratic: a reproducible sparse
// attention mixer", section Finite-range scaling (fixed candidate slots).

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mdr {

constexpr int kRouteWarps = 4;

__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const RouteArgs a) {
  extern __shared__ int32_t rsmem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nprobe = [&] { int n = 1; for (int s = 0; s < a.P; ++s) n *= a.probes; return n; }();
  const int cmax = nprobe * a.cap;
  int32_t* cand = rsmem + warp * 2 * cmax;
  float* score = reinterpret_cast<float*>(cand + cmax);

  const long long route = static_cast<long long>(blockIdx.x) * kRouteWarps + warp;
  const long long nroutes = static_cast<long long>(a.B) * a.Hq * a.nb;
  if (route >= nroutes) return;
  const int j = static_cast<int>(route % a.nb);
  const int hq = static_cast<int>((route / a.nb) % a.Hq);
  const int b = static_cast<int>(route / (static_cast<long long>(a.nb) * a.Hq));
  const int hkv = hq / (a.Hq / a.Hkv);
  const long long bh = static_cast<long long>(b) * a.Hkv + hkv;

  // Query summary: lane holds coordinates lane + 32 m.
  float qv[4];
  const float* qb = a.qbar + route * a.D;
  const int dm = a.D / 32;
#pragma unroll
  for (int m = 0; m < 4; ++m) qv[m] = m < dm ? qb[lane + 32 * m] : 0.f;

  // Candidates in slot order.
  const int32_t* qc = a.qcodes + route * a.P * a.probes;
  const int32_t* lists = a.lists + bh * a.A * a.cap;
  int n = 0;
  const int last = j - a.L;                        // highest eligible block
  for (int pr = 0; pr < nprobe; ++pr) {
    int ad = 0, rem = pr, div = nprobe;
    for (int s = 0; s < a.P; ++s) {
      div /= a.probes;
      const int rank = rem / div;
      rem -= rank * div;
      ad = ad * a.K + qc[s * a.probes + rank];
    }
    int cnt = a.load[bh * a.A + ad];
    cnt = cnt < a.cap ? cnt : a.cap;
    const int32_t* lst = lists + static_cast<long long>(ad) * a.cap;
    for (int base = 0; base < cnt; base += 32) {
      const int e = base + lane;
      const int id = e < cnt ? lst[e] : INT_MAX;
      const bool ok = id <= last;
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) cand[n + __popc(m & ((1u << lane) - 1u))] = id;
      n += __popc(m);
      if (__ballot_sync(0xffffffffu, e < cnt && !ok)) break;   // ascending ids: the rest are later
    }
  }
  __syncwarp();

  // Rerank.
  const float* kb = a.kbar + bh * a.nb * a.D;
  for (int c = 0; c < n; ++c) {
    const float* kr = kb + static_cast<long long>(cand[c]) * a.D;
    float acc = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (m < dm) acc = __fmaf_rn(qv[m], kr[lane + 32 * m], acc);
    acc = warp_sum(acc);
    if (lane == 0) score[c] = acc;
  }
  __syncwarp();

  // Top R: R rounds of a warp-wide best, removing the winner each time.
  int mine = INT_MAX;                               // lane r keeps the r-th winner
  for (int r = 0; r < a.R; ++r) {
    float bs = -INFINITY;
    int bi = INT_MAX, bc = -1;
    for (int c = lane; c < n; c += 32) {
      const int id = cand[c];
      if (id >= 0 && better(score[c], id, bs, bi)) { bs = score[c]; bi = id; bc = c; }
    }
    float ws = bs;
    int wi = bi;
    warp_best(ws, wi);
    if (wi == INT_MAX) break;
    if (bi == wi && bc >= 0) cand[bc] = -1;
    if (lane == r) mine = wi;
    __syncwarp();
  }

  // Remote ids ascending (-1 pads last), then the local blocks.
  int32_t* out = a.sel + route * (a.R + a.L);
  if (lane < a.R) {
    int rank = 0;
    const unsigned rmask = a.R >= 32 ? 0xffffffffu : ((1u << a.R) - 1u);
    for (int l = 0; l < a.R; ++l) {
      const int o = __shfl_sync(rmask, mine, l, 32);
      rank += (o < mine) || (o == mine && l < lane);
    }
    out[rank] = mine == INT_MAX ? -1 : mine;
  }
  if (lane < a.L) {
    const int id = j - a.L + 1 + lane;
    out[a.R + lane] = id >= 0 ? id : -1;
  }
  if (a.ncand && lane == 0) a.ncand[route] = n;
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t st) {
  int nprobe = 1;
  for (int s = 0; s < a.P; ++s) nprobe *= a.probes;
  const size_t smem = static_cast<size_t>(kRouteWarps) * 2 * nprobe * a.cap * sizeof(int32_t);
  cudaError_t e = cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long nroutes = static_cast<long long>(a.B) * a.Hq * a.nb;
  const unsigned grid = static_cast<unsigned>((nroutes + kRouteWarps - 1) / kRouteWarps);
  route_kernel<<<grid, kRouteWarps * 32, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace mdr
