// K6: one decode step -- token t of every sequence -- with an incremental
// index on a caller-owned state.
//
// The pages leave decoding open; they ask that a deployed decoder update its
// routing structures as tokens arrive while keeping causality ("Monodratic
// Claims Learned Routing Can Make Sparse Causal Attention More Selective",
// on what a deployed decoder must do), which the bounded lists make O(1).
// The reading taken here: a block enters the index when its last token
// arrives, summarised, addressed and appended to its list exactly as the
// batch build would (so a decoder and a prefill of the same prefix hold the
// same lists); the new token is routed by its own rotated query (a block of
// one token) and attends causally over the selected tokens.
//
// Three kernels, chained by programmatic dependent launch (the key kernel
// lets the route kernel start at once, so the query's rotation and probe
// codes, which need nothing the key kernel writes, overlap it):
//   decode_keys_kernel    one CTA per (b, KV head): rotate k_t into the key
//                         cache, copy v_t, add the rotated key (float32) to
//                         the running sum of the block; when t completes its
//                         block: the block mean (the summary), its codes
//                         (float32 scores, highest score, lowest index) and
//                         address, and the O(1) list append (stored when the
//                         list holds fewer than cap blocks; load, overflow
//                         and maximum load updated).
//   decode_route_kernel   one CTA per (b, query head), eight warps: rotate
//                         q_t; probe codes of each subspace (top p, best
//                         first); route (warp 0): all probes' list lengths at
//                         once, slots read 32 at a time and filtered to
//                         i <= j - L; candidates scored <q'_t, kbar_i> in
//                         float32 by all warps; top R (higher score, lower
//                         id) by one ranking pass over at most 32
//                         candidates, else by rounds of warp arg-max;
//                         remote ids ascending, then the locals.
//   decode_partial_kernel one CTA per (b, query head, selected block): the
//                         block's tokens s <= t with a float32 online softmax
//                         (split-K over the selected blocks, so that a
//                         single token's gathers run on many SMs at once);
//                         the last CTA of a (b, query head) merges the blocks'
//                         (max, sum, output) in slot order into the output.

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

constexpr int kKeyThreads = 128;
constexpr int kAttWarps = 8;
constexpr int kMaxCand = 4096;           // probes^P * cap

// Order-preserving map of a float32 (not NaN) to uint32; no float maps to 0.
__device__ __forceinline__ uint32_t dec_ordered(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <typename T> __device__ __forceinline__ float ld_f(const T* p);
template <> __device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <> __device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ T st_f(float x);
template <> __device__ __forceinline__ float st_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 st_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// 16 bytes of a row (4 float32 or 8 bf16 coordinates) as floats.
template <typename T> struct Row16;
template <> struct Row16<float> {
  static constexpr int kN = 4;
  static __device__ __forceinline__ void unpack(const uint4& r, float* o) {
    o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
    o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
  }
};
template <> struct Row16<__nv_bfloat16> {
  static constexpr int kN = 8;
  static __device__ __forceinline__ void unpack(const uint4& r, float* o) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      o[2 * i] = __uint_as_float(w[i] << 16);             // the element at the lower address
      o[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

// Score of codeword k of subspace sdx against xs (dsub floats, shared
// memory): four float32 partial sums over d mod 4, added pairwise.
__device__ __forceinline__ float codeword_score(const float* xs, const float* codebooks, int sdx, int k, int K,
                                                int dsub) {
  const float4* cw = reinterpret_cast<const float4*>(codebooks + (static_cast<size_t>(sdx) * K + k) * dsub);
  const float4* x4 = reinterpret_cast<const float4*>(xs);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int c0 = 0; c0 < dsub / 4; c0 += 8) {      // eight row loads in flight (dsub/4 is a power of two)
    float4 cv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + u < dsub / 4) cv[u] = __ldg(cw + c0 + u);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (c0 + u < dsub / 4) {
        const float4 xv = x4[c0 + u];
        a0 = __fmaf_rn(xv.x, cv[u].x, a0);
        a1 = __fmaf_rn(xv.y, cv[u].y, a1);
        a2 = __fmaf_rn(xv.z, cv[u].z, a2);
        a3 = __fmaf_rn(xv.w, cv[u].w, a3);
      }
  }
  const float v = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
  return v == v ? v : -INFINITY;
}

// The same score with the codeword row in shared memory (rows padded to
// dsub + 4 words, so that 32 lanes reading 32 codewords hit distinct banks).
__device__ __forceinline__ float codeword_score_s(const float* xs, const float* cw_row, int dsub) {
  const float4* cw = reinterpret_cast<const float4*>(cw_row);
  const float4* x4 = reinterpret_cast<const float4*>(xs);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int c = 0; c < dsub / 4; ++c) {
    const float4 xv = x4[c], cv = cw[c];
    a0 = __fmaf_rn(xv.x, cv.x, a0);
    a1 = __fmaf_rn(xv.y, cv.y, a1);
    a2 = __fmaf_rn(xv.z, cv.z, a2);
    a3 = __fmaf_rn(xv.w, cv.w, a3);
  }
  const float v = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
  return v == v ? v : -INFINITY;
}

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kKeyThreads)
decode_keys_kernel(const __grid_constant__ DecodeArgs a) {
  __shared__ __align__(16) float mean[128];
  __shared__ uint32_t wkey[kKeyThreads / 32];
  __shared__ int widx[kKeyThreads / 32];
  __shared__ int code[4];
  grid_dependency_wait();
  grid_launch_dependents();          // the route kernel rotates its query and probes meanwhile
  const int b = blockIdx.x / a.Hkv, h = blockIdx.x % a.Hkv;
  const int D = a.D, half = D / 2, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h;
  const size_t row = (static_cast<size_t>(b) * a.S + a.t) * a.Hkv + h;      // cache row of token t
  const T* kt = static_cast<const T*>(a.k_t) + bh * D;
  const T* vt = static_cast<const T*>(a.v_t) + bh * D;
  T* kc = static_cast<T*>(a.krot) + row * D;
  T* vc = static_cast<T*>(a.v) + row * D;
  float* ks = a.ksum + bh * D;
  const bool last = (a.t + 1) % a.bs == 0;
  const float inv_bs = 1.0f / static_cast<float>(a.bs);   // bs is a power of two
  for (int i = tid; i < half; i += kKeyThreads) {
    const float ang = __fmul_rn(static_cast<float>(a.t), a.inv_freq[i]);
    float sn, cs;
    sincosf(ang, &sn, &cs);
    const float x1 = ld_f(kt + i), x2 = ld_f(kt + i + half);
    const float y1 = __fmaf_rn(x1, cs, -__fmul_rn(x2, sn));
    const float y2 = __fmaf_rn(x2, cs, __fmul_rn(x1, sn));
    kc[i] = st_f<T>(y1);
    kc[i + half] = st_f<T>(y2);
    const float s1 = __fadd_rn(ks[i], y1), s2 = __fadd_rn(ks[i + half], y2);
    if (last) {
      mean[i] = s1 * inv_bs;
      mean[i + half] = s2 * inv_bs;
      ks[i] = 0.f;
      ks[i + half] = 0.f;
    } else {
      ks[i] = s1;
      ks[i + half] = s2;
    }
  }
  for (int i = tid; i < D; i += kKeyThreads) vc[i] = vt[i];
  if (!last) return;

  // Block j is complete: summary, codes, address, append.
  __syncthreads();
  const int j = a.t / a.bs, dsub = D / a.P;
  float* kb = a.kbar + (bh * a.nb + j) * D;
  for (int i = tid; i < D; i += kKeyThreads) kb[i] = mean[i];
  for (int sdx = 0; sdx < a.P; ++sdx) {
    const uint32_t key = tid < a.K ? dec_ordered(codeword_score(mean + sdx * dsub, a.codebooks, sdx, tid, a.K, dsub)) : 0u;
    const uint32_t top = __reduce_max_sync(0xffffffffu, key);
    const uint32_t lo = __reduce_min_sync(0xffffffffu, key == top ? static_cast<uint32_t>(tid) : 0xffffffffu);
    if (lane == 0) { wkey[warp] = top; widx[warp] = static_cast<int>(lo); }
    __syncthreads();
    if (tid == 0) {
      uint32_t bk = wkey[0];
      int bi = widx[0];
      for (int w = 1; w < kKeyThreads / 32; ++w)
        if (wkey[w] > bk) { bk = wkey[w]; bi = widx[w]; }      // warps in index order: ties keep the lower
      code[sdx] = bi;
    }
    __syncthreads();
  }
  if (tid == 0) {
    int ad = 0;
    for (int sdx = 0; sdx < a.P; ++sdx) ad = ad * a.K + code[sdx];
    a.addr[bh * a.nb + j] = ad;
    int32_t* ld = a.load + bh * a.A + ad;
    const int pos = *ld;
    if (pos < a.cap) a.lists[(bh * a.A + ad) * a.cap + pos] = j;
    *ld = pos + 1;
    if (pos >= a.cap) a.overflow[bh] += 1;
    if (pos + 1 > a.maxload[bh]) a.maxload[bh] = pos + 1;
  }
}

// Shared memory of decode_route_kernel, in 4-byte words.
constexpr int kDecQ = 0;                          // rotated query [D <= 128]
constexpr int kDecCode = kDecQ + 128;             // probe codes [P * probes <= 64]
constexpr int kDecPAddr = kDecCode + 64;          // probed addresses [<= 64]
constexpr int kDecOffs = kDecPAddr + 64;          // slot offsets [<= 65]
constexpr int kDecCand = kDecOffs + 68;          // candidate ids [kMaxCand]
constexpr int kDecKey = kDecCand + kMaxCand;      // candidate score keys [kMaxCand]
constexpr int kDecWords = kDecKey + kMaxCand;    // then the codebooks [P][K][dsub + 4]

template <typename T>
__global__ void __launch_bounds__(kAttWarps * 32)
decode_route_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(16) float dsm[];
  float* qs = dsm + kDecQ;
  int* pcode = reinterpret_cast<int*>(dsm + kDecCode);
  int* paddr = reinterpret_cast<int*>(dsm + kDecPAddr);
  int* offs = reinterpret_cast<int*>(dsm + kDecOffs);
  int* cand = reinterpret_cast<int*>(dsm + kDecCand);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(dsm + kDecKey);
  __shared__ int s_ncand;
  const int b = blockIdx.x / a.Hq, hq = blockIdx.x % a.Hq, h = hq / (a.Hq / a.Hkv);
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h, bq = static_cast<size_t>(b) * a.Hq + hq;
  const int t = a.t, j = t / a.bs, D = a.D, half = D / 2, dsub = D / a.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // 0. the codebooks into shared memory (an input: no wait needed); the
  // barrier after the rotation covers these stores too.
  float* cbs = dsm + kDecWords;
  {
    const int dsub0 = D / a.P, RS = dsub0 + 4;
    const float4* cb4 = reinterpret_cast<const float4*>(a.codebooks);
    for (int i4 = tid; i4 < a.P * a.K * dsub0 / 4; i4 += kAttWarps * 32) {
      const int i = 4 * i4, row = i / dsub0, d = i - row * dsub0;   // row = sdx * K + k
      *reinterpret_cast<float4*>(cbs + row * RS + d) = cb4[i4];
    }
  }

  // 1. rotated query.
  const T* qt = static_cast<const T*>(a.q_t) + bq * D;
  for (int i = tid; i < half; i += kAttWarps * 32) {
    const float ang = __fmul_rn(static_cast<float>(t), a.inv_freq[i]);
    float sn, cs;
    sincosf(ang, &sn, &cs);
    const float x1 = ld_f(qt + i), x2 = ld_f(qt + i + half);
    qs[i] = __fmaf_rn(x1, cs, -__fmul_rn(x2, sn));
    qs[i + half] = __fmaf_rn(x2, cs, __fmul_rn(x1, sn));
  }
  __syncthreads();

  // 2. probe codes: warp sdx, lane = codeword (K <= 128), top p best first.
  if (warp < a.P) {
    const int sdx = warp;
    uint32_t key[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int k = lane + 32 * m;
      key[m] = k < a.K ? dec_ordered(codeword_score_s(qs + sdx * dsub, cbs + (sdx * a.K + k) * (dsub + 4), dsub)) : 0u;
    }
    for (int rnd = 0; rnd < a.probes; ++rnd) {
      uint32_t lk = key[0];
      int lm = 0;
#pragma unroll
      for (int m = 1; m < 4; ++m)
        if (key[m] > lk) { lk = key[m]; lm = m; }
      const uint32_t top = __reduce_max_sync(0xffffffffu, lk);
      const int bi = static_cast<int>(
          __reduce_min_sync(0xffffffffu, lk == top ? static_cast<uint32_t>(lane + 32 * lm) : 0xffffffffu));
      if (lane == 0) pcode[sdx * a.probes + rnd] = bi;
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (lane + 32 * m == bi) key[m] = 0u;
    }
  }
  __syncthreads();
  // Steps 1 and 2 read only the step's query and the codebooks; from here on
  // the index, which the key kernel of this step may have appended to.
  grid_dependency_wait();

  // 3. route (warp 0).
  if (warp == 0) {
    int nprobe = 1;
    for (int s = 0; s < a.P; ++s) nprobe *= a.probes;
    const int32_t* lists = a.lists + bh * a.A * a.cap;
    const int32_t* load = a.load + bh * a.A;
    const int last = j - a.L;                     // highest eligible block
    int c[2] = {0, 0};
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int pr = lane + 32 * hh;
      if (pr < nprobe) {
        int ad = 0, rem = pr, div = nprobe;
        for (int s = 0; s < a.P; ++s) {           // first subspace's rank slowest
          div /= a.probes;
          const int rank = rem / div;
          rem -= rank * div;
          ad = ad * a.K + pcode[s * a.probes + rank];
        }
        paddr[pr] = ad;
        const int cl = load[ad];
        c[hh] = cl < a.cap ? cl : a.cap;
      }
    }
    int s0 = c[0], s1 = c[1];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u0 = __shfl_up_sync(0xffffffffu, s0, o), u1 = __shfl_up_sync(0xffffffffu, s1, o);
      if (lane >= o) { s0 += u0; s1 += u1; }
    }
    const int t0 = __shfl_sync(0xffffffffu, s0, 31);
    const int total = t0 + __shfl_sync(0xffffffffu, s1, 31);
    if (lane < nprobe) offs[lane] = s0 - c[0];
    if (lane + 32 < nprobe) offs[lane + 32] = t0 + s1 - c[1];
    if (lane == 0) offs[nprobe] = total;
    __syncwarp();
    int n = 0;
    for (int base = 0; base < total; base += 32) {
      const int e = base + lane;
      int id = INT_MAX;
      if (e < total) {
        int lo = 0, hi = nprobe - 1;              // probe p with offs[p] <= e < offs[p+1]
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (offs[mid] <= e) lo = mid; else hi = mid - 1;
        }
        id = lists[static_cast<size_t>(paddr[lo]) * a.cap + (e - offs[lo])];
      }
      const bool ok = id >= 0 && id <= last;
      const unsigned m = __ballot_sync(0xffffffffu, ok);
      if (ok) cand[n + __popc(m & ((1u << lane) - 1u))] = id;
      n += __popc(m);
    }
    if (lane == 0) s_ncand = n;
  }
  __syncthreads();

  // Candidate scores <q'_t, kbar_i>, float32, by all warps: warp w takes
  // candidates w, w + 8, ..., four rows in flight; a lane holds D/32
  // coordinates (in order), the lanes' partial sums meet in a fixed butterfly.
  {
    const int n = s_ncand, vpl = D / 32;
    const float* kb = a.kbar + bh * a.nb * D;
    float qv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = e < vpl ? qs[lane * vpl + e] : 0.f;
    for (int c0 = warp; c0 < n; c0 += 4 * kAttWarps) {
      float sc[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int ci = c0 + x * kAttWarps;
        float kv[4] = {0.f, 0.f, 0.f, 0.f};
        if (ci < n) {
          const float* kr = kb + static_cast<size_t>(cand[ci]) * D + lane * vpl;
          if (vpl == 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(kr));
            kv[0] = f.x; kv[1] = f.y; kv[2] = f.z; kv[3] = f.w;
          } else if (vpl == 2) {
            const float2 f = __ldg(reinterpret_cast<const float2*>(kr));
            kv[0] = f.x; kv[1] = f.y;
          } else {
            kv[0] = __ldg(kr);
          }
        }
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc = __fmaf_rn(qv[e], kv[e], acc);
        sc[x] = acc;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int x = 0; x < 4; ++x) sc[x] = __fadd_rn(sc[x], __shfl_xor_sync(0xffffffffu, sc[x], off));
      if (lane == 0)
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int ci = c0 + x * kAttWarps;
          if (ci < n) ckey[ci] = dec_ordered(sc[x] == sc[x] ? sc[x] : -INFINITY);
        }
    }
  }
  __syncthreads();

  if (warp == 0 && s_ncand <= 32) {
    // At most 32 candidates: lane l ranks candidate l against all the others
    // in one pass (higher score first, lower id on equal scores); the best R
    // are written in ascending id order, -1 after them -- the same selection
    // as the rounds below, without their chain of dependent reductions.
    const int n = s_ncand;
    const bool have = lane < n;
    const uint32_t k = have ? ckey[lane] : 0u;
    const int id = have ? cand[lane] : INT_MAX;
    int better = 0;
    for (int m = 0; m < n; ++m) {
      const uint32_t km = __shfl_sync(0xffffffffu, k, m);
      const int im = __shfl_sync(0xffffffffu, id, m);
      better += (km > k || (km == k && im < id)) ? 1 : 0;
    }
    const bool win = have && better < a.R;
    const unsigned wmask = __ballot_sync(0xffffffffu, win);
    int pos = 0;                                  // winners with a lower id
    for (int m = 0; m < n; ++m) {
      const int im = __shfl_sync(0xffffffffu, id, m);
      pos += (((wmask >> m) & 1u) && im < id) ? 1 : 0;
    }
    int32_t* srow = a.sel_t + bq * (a.R + a.L);
    const int nwin = __popc(wmask);
    if (win) srow[pos] = id;
    if (lane >= nwin && lane < a.R) srow[lane] = -1;
    if (lane < a.L) {
      const int lid = j - a.L + 1 + lane;
      srow[a.R + lane] = lid >= 0 ? lid : -1;
    }
    if (a.ncand_t && lane == 0) a.ncand_t[bq] = n;
  } else if (warp == 0) {
    const int n = s_ncand;
    int mine = INT_MAX;                           // lane r: the r-th winner
    for (int r = 0; r < a.R; ++r) {
      uint32_t lk = 0u;
      int lid = INT_MAX, lc = -1;
      for (int ci = lane; ci < n; ci += 32) {
        const uint32_t k = ckey[ci];
        const int id = cand[ci];
        if (k > lk || (k == lk && k != 0u && id < lid)) { lk = k; lid = id; lc = ci; }
      }
      const uint32_t top = __reduce_max_sync(0xffffffffu, lk);
      if (top == 0u) break;
      const int wid = static_cast<int>(
          __reduce_min_sync(0xffffffffu, lk == top ? static_cast<uint32_t>(lid) : 0xffffffffu));
      if (lk == top && lid == wid) ckey[lc] = 0u;
      __syncwarp();
      if (lane == r) mine = wid;
    }
    int32_t* srow = a.sel_t + bq * (a.R + a.L);
    int rank = 0;
    if (a.R > 0) {
      for (int l = 0; l < a.R; ++l) {
        const int o = __shfl_sync(0xffffffffu, mine, l);
        rank += (o < mine) || (o == mine && l < lane);
      }
    }
    if (lane < a.R) srow[rank] = mine == INT_MAX ? -1 : mine;
    if (lane < a.L) {
      const int id = j - a.L + 1 + lane;
      srow[a.R + lane] = id >= 0 ? id : -1;
    }
    if (a.ncand_t && lane == 0) a.ncand_t[bq] = n;
  }
  // The rotated query, for the attention kernel of this step.
  for (int i = tid; i < D; i += kAttWarps * 32) a.qrot_t[bq * D + i] = qs[i];
}

// Attention of token t over one selected block: CTA (b*Hq + hq, slot) takes
// block sel[slot] (tokens s <= t).  A row of the cache is read as 16-byte
// pieces by kLpr consecutive lanes, so a warp reads 32/kLpr rows per load
// and each lane keeps eight loads of K and eight of V in flight at once (one
// memory round trip per 8*32/kLpr rows).  Scores are summed over the lanes
// of a row; the warp shares one running maximum (float32 online softmax) and
// each lane accumulates its coordinates over its own rows; the row groups of
// a warp, then the four warps, are merged into the block's (max, sum,
// output).  The last CTA of a (b, hq) to finish merges all blocks, in slot
// order, into the output, reading every block's partial result in one
// parallel round.
// Five CTAs per SM (96 registers): more blocks' loads in flight per SM.
template <typename T, int kLpr>
__global__ void __launch_bounds__(128, 5)
decode_partial_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int kEpl = Row16<T>::kN;       // coordinates per lane
  constexpr int kRpi = 32 / kLpr;          // rows per warp load
  constexpr int kSteps = 8;                // loads of K (and of V) in flight per lane
  constexpr int kRowsWarp = kSteps * kRpi;
  constexpr int kRowsPass = 4 * kRowsWarp;
  constexpr int kMaxSlots = 64;            // R + L <= 64 (the configuration check)
  __shared__ float wm[4], wl[4];
  __shared__ float wo[4][128];
  __shared__ float s_m[kMaxSlots], s_l[kMaxSlots], s_f[kMaxSlots];
  __shared__ int s_last;
  grid_dependency_wait();            // sel and the rotated query of this step
  const int bq = blockIdx.x, slot = blockIdx.y, nsl = a.R + a.L;
  const int b = bq / a.Hq, hq = bq % a.Hq, h = hq / (a.Hq / a.Hkv);
  const int t = a.t, D = a.D;        // D == kLpr * kEpl
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane / kLpr, col = (lane % kLpr) * kEpl;
  const int blk = a.sel_t[static_cast<size_t>(bq) * nsl + slot];
  float m = -INFINITY, l = 0.f, o[kEpl];
#pragma unroll
  for (int e = 0; e < kEpl; ++e) o[e] = 0.f;
  if (blk >= 0) {
    const int first = blk * a.bs, ntok = min(a.bs, t + 1 - first);
    float qv[kEpl];
#pragma unroll
    for (int e = 0; e < kEpl; ++e) qv[e] = a.qrot_t[static_cast<size_t>(bq) * D + col + e] * a.scale;
    const size_t rs = static_cast<size_t>(a.Hkv) * D;                 // elements from one token to the next
    const size_t base = (static_cast<size_t>(b) * a.S + first) * rs + static_cast<size_t>(h) * D + col;
    const T* kb = static_cast<const T*>(a.krot) + base;
    const T* vb = static_cast<const T*>(a.v) + base;
    for (int r0 = 0; r0 < ntok; r0 += kRowsPass) {
      const int rw = r0 + warp * kRowsWarp + grp;                      // row of step 0; step s adds s*kRpi
      uint4 kr[kSteps], vr[kSteps];
#pragma unroll
      for (int s = 0; s < kSteps; ++s) {
        const int r = rw + s * kRpi;
        if (r < ntok) {
          kr[s] = *reinterpret_cast<const uint4*>(kb + r * rs);
          vr[s] = *reinterpret_cast<const uint4*>(vb + r * rs);
        } else {
          kr[s] = make_uint4(0u, 0u, 0u, 0u);
          vr[s] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      float sc[kSteps];
#pragma unroll
      for (int s = 0; s < kSteps; ++s) {
        float kf[kEpl];
        Row16<T>::unpack(kr[s], kf);
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < kEpl; ++e) d = __fmaf_rn(qv[e], kf[e], d);
        sc[s] = d;
      }
#pragma unroll
      for (int off = kLpr / 2; off > 0; off >>= 1)
#pragma unroll
        for (int s = 0; s < kSteps; ++s) sc[s] = __fadd_rn(sc[s], __shfl_xor_sync(0xffffffffu, sc[s], off));
      float pm = -INFINITY;
#pragma unroll
      for (int s = 0; s < kSteps; ++s) {
        if (rw + s * kRpi >= ntok) sc[s] = -INFINITY;
        pm = fmaxf(pm, sc[s]);
      }
#pragma unroll
      for (int off = kLpr; off < 32; off <<= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, off));
      if (pm == -INFINITY) break;      // warp-uniform: this warp has no row left in the block
      const float mn = fmaxf(m, pm);
      const float alpha = expf(m - mn);
      l *= alpha;
#pragma unroll
      for (int e = 0; e < kEpl; ++e) o[e] *= alpha;
#pragma unroll
      for (int s = 0; s < kSteps; ++s) {
        const float p = expf(sc[s] - mn);
        l += p;
        float vf[kEpl];
        Row16<T>::unpack(vr[s], vf);
#pragma unroll
        for (int e = 0; e < kEpl; ++e) o[e] = __fmaf_rn(p, vf[e], o[e]);
      }
      m = mn;
    }
    // The warp's row groups share m: add their sums and outputs.
#pragma unroll
    for (int off = kLpr; off < 32; off <<= 1) {
      l = __fadd_rn(l, __shfl_xor_sync(0xffffffffu, l, off));
#pragma unroll
      for (int e = 0; e < kEpl; ++e) o[e] = __fadd_rn(o[e], __shfl_xor_sync(0xffffffffu, o[e], off));
    }
  }
  if (lane == 0) { wm[warp] = m; wl[warp] = l; }
  if (lane < kLpr) {
#pragma unroll
    for (int e = 0; e < kEpl; ++e) wo[warp][col + e] = o[e];
  }
  __syncthreads();
  // This block's (max, sum, output) over its four warps.
  float* pp = a.part + (static_cast<size_t>(bq) * nsl + slot) * (2 + D);
  float M = -INFINITY;
  for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w]);
  for (int i = tid; i < D; i += 128) {
    float num = 0.f;
    for (int w = 0; w < 4; ++w)
      if (wm[w] != -INFINITY) num = __fmaf_rn(expf(wm[w] - M), wo[w][i], num);
    pp[2 + i] = num;
  }
  if (tid == 0) {
    float den = 0.f;
    for (int w = 0; w < 4; ++w)
      if (wm[w] != -INFINITY) den = __fmaf_rn(expf(wm[w] - M), wl[w], den);
    pp[0] = M;
    pp[1] = den;
  }
  // Publish: the barrier orders the CTA's stores before thread 0's fence
  // and counter increment (a release, cumulative over the barrier); the last
  // block's thread 0 fences again (acquire) before the barrier after which
  // its threads read the other blocks' partial results.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s_last = atomicAdd(a.done + bq, 1) == nsl - 1;
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  // Last block of this (b, hq): every block's max and sum in one round, then
  // the outputs weighted in slot order.
  const float* pb = a.part + static_cast<size_t>(bq) * nsl * (2 + D);
  if (tid < nsl) {
    s_m[tid] = __ldcg(pb + tid * (2 + D));
    s_l[tid] = __ldcg(pb + tid * (2 + D) + 1);
  }
  __syncthreads();
  float MM = -INFINITY;
  for (int s = 0; s < nsl; ++s) MM = fmaxf(MM, s_m[s]);
  if (tid < nsl) s_f[tid] = s_m[tid] == -INFINITY ? 0.f : expf(s_m[tid] - MM);
  __syncthreads();
  float den = 0.f;
  for (int s = 0; s < nsl; ++s) den = __fmaf_rn(s_f[s], s_l[s], den);
  T* out = static_cast<T*>(a.out_t) + static_cast<size_t>(bq) * D;
  for (int i = tid; i < D; i += 128) {
    float num = 0.f;
#pragma unroll 8
    for (int s = 0; s < nsl; ++s) num = __fmaf_rn(s_f[s], __ldcg(pb + s * (2 + D) + 2 + i), num);
    out[i] = st_f<T>(num / den);
  }
  if (tid == 0) a.done[bq] = 0;
}

template <typename T>
cudaError_t launch_partial(const DecodeArgs& a, cudaStream_t st) {
  const dim3 grid(a.B * a.Hq, a.R + a.L);
  const int lpr = a.D * static_cast<int>(sizeof(T)) / 16;   // lanes per row (D is 32, 64 or 128)
  if (lpr == 8) return launch_pdl(decode_partial_kernel<T, 8>, grid, dim3(128), 0, st, a);
  if (lpr == 16) return launch_pdl(decode_partial_kernel<T, 16>, grid, dim3(128), 0, st, a);
  if constexpr (sizeof(T) == 4) {
    if (lpr == 32) return launch_pdl(decode_partial_kernel<T, 32>, grid, dim3(128), 0, st, a);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  if (a.D > 128 || a.D % 32 != 0 || a.K > 128 || a.P > 4 || a.R + a.L > 64) return cudaErrorInvalidValue;
  cudaError_t e = bf16 ? launch_pdl(decode_keys_kernel<__nv_bfloat16>, dim3(a.B * a.Hkv), dim3(kKeyThreads), 0, st, a)
                       : launch_pdl(decode_keys_kernel<float>, dim3(a.B * a.Hkv), dim3(kKeyThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  const size_t smem = (static_cast<size_t>(kDecWords) + static_cast<size_t>(a.K) * (a.D + 4 * a.P)) * sizeof(float);
  void (*k)(DecodeArgs) = bf16 ? decode_route_kernel<__nv_bfloat16> : decode_route_kernel<float>;
  if ((e = cached_allow_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem))) != cudaSuccess) return e;
  if ((e = launch_pdl(k, dim3(a.B * a.Hq), dim3(kAttWarps * 32), smem, st, a)) != cudaSuccess) return e;
  if ((e = bf16 ? launch_partial<__nv_bfloat16>(a, st) : launch_partial<float>(a, st)) != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
