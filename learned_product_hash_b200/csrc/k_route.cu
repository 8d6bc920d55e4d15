// K4: probe -> fixed candidate slots -> rerank -> top-R, plus L local blocks.
//
// One warp per route (sequence b, query head hq, query block j).  The probed
// addresses are the product of the p best codewords of each subspace (first
// subspace's rank slowest).  Each probed address owns cap candidate slots:
// the stored blocks of its list that are remote-eligible, i <= j - L.  The
// lanes look up all probes' list lengths at once, prefix-sum them into slot
// offsets, and read the stored slots 32 at a time, so a route costs a few
// dependent memory round trips, not one per probe.  Candidates are scored by
// <qbar_j, kbar_i> in float32: the D/4 lanes of a lane group read a
// candidate's row together (one coalesced 16-byte read each, several
// candidates in flight) and add their four-term partial sums with a fixed
// butterfly.  Batches of at most 224 candidates are merged into the running
// top R (higher score first, lower id on equal scores): by rank counting
// when the batch and the winners are at most 64, else by R rounds of warp
// arg-max.  The R winners are written in ascending id order, -1 padded; then
// the local blocks j-L+1..j.
//
// Forced-target diagnostic ("Why Learned Product-Hash Routing Matters Now":
// the labelled target block is put into the selected set under the same
// attention budget): a forced id f with 0 <= f <= j - L seeds the running
// winners with score +inf, and f is left out of the probed candidates, so
// the R winners are f and the R - 1 best others -- f replaces the weakest
// choice when routing missed it and changes nothing when routing found it.
// Any other forced value leaves the route unchanged; ncand still counts the
// eligible candidates the probes found.
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

// Candidates are scored and merged into the running top R in batches of at
// most kBatch, so a warp's shared memory does not grow with probes^P * cap.
constexpr int kBatch = 224;
// Shared memory of one warp, in 4-byte words: the query summary (D <= 128),
// probe addresses (64), slot offsets (65, padded to 68), candidate ids and
// scores (kBatch + 32 each: a batch, then the running winners).
constexpr int kRouteWarpWords = 128 + 64 + 68 + 2 * (kBatch + 32);

template <bool kForced>
__global__ void __launch_bounds__(kRouteWarps * 32)
route_kernel(const RouteArgs a) {
  extern __shared__ int32_t rsmem[];
  grid_dependency_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int nprobe = 1;
  for (int s = 0; s < a.P; ++s) nprobe *= a.probes;
  int32_t* wsm = rsmem + warp * kRouteWarpWords;
  float* qs = reinterpret_cast<float*>(wsm);
  int32_t* paddr = wsm + 128;
  int32_t* offs = paddr + 64;
  int32_t* cand = offs + 68;                       // [kBatch) batch, [kBatch, kBatch+R) winners
  float* score = reinterpret_cast<float*>(cand + kBatch + 32);

  const int nbr = a.nbr > 0 ? a.nbr : a.nb;         // query blocks a.j0 .. a.j0 + nbr - 1
  const long long rl = static_cast<long long>(blockIdx.x) * kRouteWarps + warp;
  if (rl >= static_cast<long long>(a.B) * a.Hq * nbr) return;
  const long long bhq = rl / nbr;
  const int j = a.j0 + static_cast<int>(rl - bhq * nbr);
  const int hq = static_cast<int>(bhq % a.Hq);
  const int b = static_cast<int>(bhq / a.Hq);
  const long long route = bhq * a.nb + j;           // (b, hq, j) in the [B,Hq,nb] grid
  const int hkv = hq / (a.Hq / a.Hkv);
  const long long bh = static_cast<long long>(b) * a.Hkv + hkv;
  const int32_t* lists = a.lists + bh * a.A * a.cap;
  const int last = j - a.L;                        // highest eligible block
  if (a.upstream_status && *reinterpret_cast<const volatile int32_t*>(a.upstream_status) != 0) {
    // The summaries this route would read may be incomplete: no route.
    for (int s = lane; s < a.R + a.L; s += 32) a.sel[route * (a.R + a.L) + s] = -1;
    if (a.ncand && lane == 0) a.ncand[route] = -1;
    return;
  }

  for (int d = lane; d < a.D; d += 32) qs[d] = a.qbar[route * a.D + d];
  int forced = kForced ? a.force[route] : -1;
  if (forced < 0 || forced > last || a.R <= 0) forced = INT_MIN;   // not a remote-eligible block

  // Probed addresses and their stored counts, all probes at once: lane l
  // owns probes l and l + 32 (first subspace's rank slowest).
  const int32_t* qc = a.qcodes + route * a.P * a.probes;
  int c0 = 0, c1 = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int pr = lane + 32 * h;
    if (pr < nprobe) {
      int ad = 0, rem = pr, div = nprobe;
      for (int s = 0; s < a.P; ++s) {
        div /= a.probes;
        const int rank = rem / div;
        rem -= rank * div;
        ad = ad * a.K + qc[s * a.probes + rank];
      }
      paddr[pr] = ad;
      const int cl = a.load[bh * a.A + ad];
      if (h == 0) c0 = cl < a.cap ? cl : a.cap;
      else c1 = cl < a.cap ? cl : a.cap;
    }
  }
  // Exclusive prefix sums of the counts give each probe's first slot.
  int s0 = c0, s1 = c1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u0 = __shfl_up_sync(0xffffffffu, s0, o);
    const int u1 = __shfl_up_sync(0xffffffffu, s1, o);
    if (lane >= o) { s0 += u0; s1 += u1; }
  }
  const int t0 = __shfl_sync(0xffffffffu, s0, 31);
  const int total = t0 + __shfl_sync(0xffffffffu, s1, 31);
  if (lane < nprobe) offs[lane] = s0 - c0;
  if (lane + 32 < nprobe) offs[lane + 32] = t0 + s1 - c1;
  if (lane == 0) offs[nprobe] = total;
  __syncwarp();

  // Read every stored slot of the probed lists, 32 per step, keep the
  // remote-eligible blocks; every kBatch of them (and at the end) score the
  // batch and merge it with the running winners.
  const float* kb = a.kbar + bh * a.nb * a.D;
  int nbuf = 0, n = 0, nwin = 0;
  int mine = INT_MAX;                              // lane r: r-th winner id
  if (kForced && forced != INT_MIN) {              // the forced block is winner 0 from the start
    if (lane == 0) {
      cand[kBatch] = forced;
      score[kBatch] = INFINITY;
      mine = forced;
    }
    nwin = 1;
    __syncwarp();
  }
  for (int base = 0; base < total; base += 32) {
    const int e = base + lane;
    int id = INT_MAX;
    if (e < total) {
      int lo = 0, hi = nprobe - 1;                 // probe p with offs[p] <= e < offs[p+1]
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offs[mid] <= e) lo = mid; else hi = mid - 1;
      }
      id = lists[static_cast<long long>(paddr[lo]) * a.cap + (e - offs[lo])];
    }
    const bool elig = id <= last;
    const bool ok = elig && (!kForced || id != forced);
    const unsigned m = __ballot_sync(0xffffffffu, ok);
    if (ok) cand[nbuf + __popc(m & ((1u << lane) - 1u))] = id;
    nbuf += __popc(m);
    n += __popc(__ballot_sync(0xffffffffu, elig));
    if (nbuf <= kBatch - 32 && base + 32 < total) continue;
    __syncwarp();
    // Score the batch: lane group g (F4 = D/4 lanes) takes candidates g,
    // g + 32/F4, ...; lane pos holds coordinates 4 pos .. 4 pos + 3.
    {
      const int F4 = a.D / 4, cpi = 32 / F4, grp = lane / F4, pos = lane % F4;
      const float4 qv = reinterpret_cast<const float4*>(qs)[pos];
      for (int c0 = 0; c0 < nbuf; c0 += 8 * cpi) {
        float pr[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u * cpi + grp;
          pr[u] = 0.f;
          if (c < nbuf) {
            const float4 kv = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(cand[c]) * a.D) + pos);
            pr[u] = __fmaf_rn(qv.w, kv.w, __fmaf_rn(qv.z, kv.z, __fmaf_rn(qv.y, kv.y, __fmul_rn(qv.x, kv.x))));
          }
        }
        // Fixed butterfly over the F4 lanes of a group (F4 in {8, 16, 32});
        // the levels are unrolled so the eight sums proceed side by side.
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float t = __shfl_xor_sync(0xffffffffu, pr[u], o);
            if (o < F4) pr[u] = __fadd_rn(pr[u], t);
          }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u * cpi + grp;
          if (pos == 0 && c < nbuf) score[c] = pr[u];
        }
      }
    }
    __syncwarp();
    // Top R of the batch and the previous winners (higher score, lower id).
    int newwin = 0;
    float myscore = -INFINITY;
    mine = INT_MAX;
    if (nbuf + nwin <= 64) {
      // Rank of entry e (batch entries, then the winners) among all of them.
      const int T = nbuf + nwin;
      int rk[2], eid[2];
      float esc[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int e = lane + 32 * h;
        rk[h] = INT_MAX;
        eid[h] = INT_MAX;
        esc[h] = -INFINITY;
        if (e < T) {
          const int ce = e < nbuf ? e : kBatch + (e - nbuf);
          eid[h] = cand[ce];
          esc[h] = score[ce];
          int r = 0;
#pragma unroll 4
          for (int f = 0; f < T; ++f) {
            const int cf = f < nbuf ? f : kBatch + (f - nbuf);
            r += better(score[cf], cand[cf], esc[h], eid[h]) ? 1 : 0;
          }
          rk[h] = r;
        }
      }
      __syncwarp();
#pragma unroll
      for (int h = 0; h < 2; ++h)
        if (rk[h] < a.R) { cand[kBatch + rk[h]] = eid[h]; score[kBatch + rk[h]] = esc[h]; }
      __syncwarp();
      newwin = T < a.R ? T : a.R;
      if (lane < newwin) { mine = cand[kBatch + lane]; myscore = score[kBatch + lane]; }
    } else {
    for (int r = 0; r < a.R; ++r) {
      float bs = -INFINITY;
      int bi = INT_MAX, bc = -1;
      for (int c = lane; c < nbuf; c += 32) {
        const int cid = cand[c];
        if (cid >= 0 && better(score[c], cid, bs, bi)) { bs = score[c]; bi = cid; bc = c; }
      }
      if (lane < nwin) {
        const int c = kBatch + lane;
        const int cid = cand[c];
        if (cid >= 0 && better(score[c], cid, bs, bi)) { bs = score[c]; bi = cid; bc = c; }
      }
      float ws = bs;
      int wi = bi;
      warp_best(ws, wi);
      if (wi == INT_MAX) break;
      if (bi == wi && bc >= 0) cand[bc] = -1;
      if (lane == r) { mine = wi; myscore = ws; }
      ++newwin;
      __syncwarp();
    }
    }
    __syncwarp();
    if (lane < newwin) { cand[kBatch + lane] = mine; score[kBatch + lane] = myscore; }
    nwin = newwin;
    nbuf = 0;
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
  const size_t smem = static_cast<size_t>(kRouteWarps) * kRouteWarpWords * sizeof(int32_t);
  const auto kern = a.force ? route_kernel<true> : route_kernel<false>;
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return cudaErrorInvalidValue;
  const long long nroutes = static_cast<long long>(a.B) * a.Hq * nbr;
  const unsigned grid = static_cast<unsigned>((nroutes + kRouteWarps - 1) / kRouteWarps);
  e = launch_pdl(kern, dim3(grid), dim3(kRouteWarps * 32), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
