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
// Two kernels, chained by programmatic dependent launch:
//   decode_keys_kernel    one CTA per (b, KV head): rotate k_t into the key
//                         cache, copy v_t, add the rotated key (float32) to
//                         the running sum of the block; when t completes its
//                         block: the block mean (the summary), its codes
//                         (float32 scores, highest score, lowest index) and
//                         address, and the O(1) list append (stored when the
//                         list holds fewer than cap blocks; load, overflow
//                         and maximum load updated).
//   decode_attend_kernel  one CTA per (b, query head), eight warps: rotate
//                         q_t; probe codes of each subspace (top p, best
//                         first); route (warp 0): all probes' list lengths at
//                         once, slots read 32 at a time and filtered to
//                         i <= j - L, candidates scored <q'_t, kbar_i> in
//                         float32, top R by rounds of warp arg-max (higher
//                         score, lower id), remote ids ascending, then the
//                         locals; attention: the selected tokens s <= t are
//                         split over the eight warps, each with a float32
//                         online softmax (lanes hold D/32 coordinates of the
//                         key and value rows it reads), merged at the end.

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

// Score of codeword k of subspace sdx against xs (dsub floats, shared
// memory): four float32 partial sums over d mod 4, added pairwise.
__device__ __forceinline__ float codeword_score(const float* xs, const float* codebooks, int sdx, int k, int K,
                                                int dsub) {
  const float4* cw = reinterpret_cast<const float4*>(codebooks + (static_cast<size_t>(sdx) * K + k) * dsub);
  const float4* x4 = reinterpret_cast<const float4*>(xs);
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  for (int d4 = 0; d4 < dsub / 4; ++d4) {
    const float4 xv = x4[d4], cv = __ldg(cw + d4);
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

// Shared memory of decode_attend_kernel, in 4-byte words.
constexpr int kDecQ = 0;                          // rotated query [D <= 128]
constexpr int kDecCode = kDecQ + 128;             // probe codes [P * probes <= 64]
constexpr int kDecPAddr = kDecCode + 64;          // probed addresses [<= 64]
constexpr int kDecOffs = kDecPAddr + 64;          // slot offsets [<= 65]
constexpr int kDecSel = kDecOffs + 68;            // selected blocks [<= 64]
constexpr int kDecTBase = kDecSel + 64;           // first token of each selected block [<= 65]
constexpr int kDecCand = kDecTBase + 68;          // candidate ids [kMaxCand]
constexpr int kDecKey = kDecCand + kMaxCand;      // candidate score keys [kMaxCand]
constexpr int kDecPart = kDecKey + kMaxCand;      // per warp: max, sum, partial output [D]
constexpr int kDecWords = kDecPart + kAttWarps * (2 + 128);

template <typename T>
__global__ void __launch_bounds__(kAttWarps * 32)
decode_attend_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(16) float dsm[];
  float* qs = dsm + kDecQ;
  int* pcode = reinterpret_cast<int*>(dsm + kDecCode);
  int* paddr = reinterpret_cast<int*>(dsm + kDecPAddr);
  int* offs = reinterpret_cast<int*>(dsm + kDecOffs);
  int* sblk = reinterpret_cast<int*>(dsm + kDecSel);
  int* tbase = reinterpret_cast<int*>(dsm + kDecTBase);
  int* cand = reinterpret_cast<int*>(dsm + kDecCand);
  uint32_t* ckey = reinterpret_cast<uint32_t*>(dsm + kDecKey);
  float* part = dsm + kDecPart;
  __shared__ int s_nsel;
  grid_dependency_wait();            // the key kernel of this step wrote token t
  const int b = blockIdx.x / a.Hq, hq = blockIdx.x % a.Hq, h = hq / (a.Hq / a.Hkv);
  const size_t bh = static_cast<size_t>(b) * a.Hkv + h, bq = static_cast<size_t>(b) * a.Hq + hq;
  const int t = a.t, j = t / a.bs, D = a.D, half = D / 2, dsub = D / a.P;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

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
      key[m] = k < a.K ? dec_ordered(codeword_score(qs + sdx * dsub, a.codebooks, sdx, k, a.K, dsub)) : 0u;
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
    __syncwarp();
    const float* kb = a.kbar + bh * a.nb * D;
    const float4* q4 = reinterpret_cast<const float4*>(qs);
    for (int ci = lane; ci < n; ci += 32) {
      const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<size_t>(cand[ci]) * D);
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = __ldg(kr + d4), qv = q4[d4];
        a0 = __fmaf_rn(qv.x, kv.x, a0);
        a1 = __fmaf_rn(qv.y, kv.y, a1);
        a2 = __fmaf_rn(qv.z, kv.z, a2);
        a3 = __fmaf_rn(qv.w, kv.w, a3);
      }
      const float v = __fadd_rn(__fadd_rn(a0, a1), __fadd_rn(a2, a3));
      ckey[ci] = dec_ordered(v == v ? v : -INFINITY);
    }
    __syncwarp();
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
    // The selected blocks for the attention: valid remote ones, then locals.
    const bool vr = lane < a.R && mine != INT_MAX;
    const unsigned mr = __ballot_sync(0xffffffffu, vr);
    if (vr) sblk[__popc(mr & ((1u << lane) - 1u))] = mine;
    const int lid = j - a.L + 1 + lane;
    const bool vl = lane < a.L && lid >= 0;
    const unsigned ml = __ballot_sync(0xffffffffu, vl);
    if (vl) sblk[__popc(mr) + __popc(ml & ((1u << lane) - 1u))] = lid;
    if (lane == 0) {
      const int ns = __popc(mr) + __popc(ml);
      int tb = 0;
      for (int i = 0; i < ns; ++i) {
        tbase[i] = tb;
        const int first = sblk[i] * a.bs;
        tb += min(a.bs, t + 1 - first);
      }
      tbase[ns] = tb;
      s_nsel = ns;
    }
  }
  __syncthreads();

  // 4. attention over the selected tokens s <= t, split over the warps.
  const int nsel = s_nsel, ntok = tbase[nsel];
  const int vpl = D / 32;                         // coordinates per lane
  float qv[4], o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    qv[e] = e < vpl ? qs[lane * vpl + e] * a.scale : 0.f;
    o[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int per = (ntok + kAttWarps - 1) / kAttWarps;
  const int u0 = warp * per, u1 = min(ntok, u0 + per);
  int bi = 0;
  for (int u = u0; u < u1; u += 4) {
    float sc[4], vv[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      sc[x] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) vv[x][e] = 0.f;
      const int uu = u + x;
      if (uu < u1) {
        while (tbase[bi + 1] <= uu) ++bi;
        const int s = sblk[bi] * a.bs + (uu - tbase[bi]);
        const size_t off = ((static_cast<size_t>(b) * a.S + s) * a.Hkv + h) * D + lane * vpl;
        const T* kr = static_cast<const T*>(a.krot) + off;
        const T* vr2 = static_cast<const T*>(a.v) + off;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (e < vpl) {
            sc[x] = __fmaf_rn(qv[e], ld_f(kr + e), sc[x]);
            vv[x][e] = ld_f(vr2 + e);
          }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int x = 0; x < 4; ++x) sc[x] = __fadd_rn(sc[x], __shfl_xor_sync(0xffffffffu, sc[x], off));
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      if (u + x >= u1) break;
      if (sc[x] > m) {
        const float alpha = expf(m - sc[x]);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] *= alpha;
        m = sc[x];
      }
      const float p = expf(sc[x] - m);
      l += p;
#pragma unroll
      for (int e = 0; e < 4; ++e) o[e] = __fmaf_rn(p, vv[x][e], o[e]);
    }
  }
  float* pw = part + warp * (2 + 128);
  if (lane == 0) { pw[0] = m; pw[1] = l; }
#pragma unroll
  for (int e = 0; e < 4; ++e)
    if (e < vpl) pw[2 + lane * vpl + e] = o[e];
  __syncthreads();
  T* out = static_cast<T*>(a.out_t) + bq * D;
  for (int i = tid; i < D; i += kAttWarps * 32) {
    float M = -INFINITY;
    for (int w = 0; w < kAttWarps; ++w) M = fmaxf(M, part[w * (2 + 128)]);
    float num = 0.f, den = 0.f;
    for (int w = 0; w < kAttWarps; ++w) {
      const float mw = part[w * (2 + 128)];
      if (mw == -INFINITY) continue;
      const float f = expf(mw - M);
      num = __fmaf_rn(f, part[w * (2 + 128) + 2 + i], num);
      den = __fmaf_rn(f, part[w * (2 + 128) + 1], den);
    }
    out[i] = st_f<T>(num / den);
  }
}

cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st) {
  if (a.D > 128 || a.D % 32 != 0 || a.K > 128 || a.P > 4) return cudaErrorInvalidValue;
  cudaError_t e = bf16 ? launch_pdl(decode_keys_kernel<__nv_bfloat16>, dim3(a.B * a.Hkv), dim3(kKeyThreads), 0, st, a)
                       : launch_pdl(decode_keys_kernel<float>, dim3(a.B * a.Hkv), dim3(kKeyThreads), 0, st, a);
  if (e != cudaSuccess) return e;
  const size_t smem = static_cast<size_t>(kDecWords) * sizeof(float);
  void (*k)(DecodeArgs) = bf16 ? decode_attend_kernel<__nv_bfloat16> : decode_attend_kernel<float>;
  if ((e = cached_allow_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem))) != cudaSuccess) return e;
  if ((e = launch_pdl(k, dim3(a.B * a.Hq), dim3(kAttWarps * 32), smem, st, a)) != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
