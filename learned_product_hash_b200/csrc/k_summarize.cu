// K1 + K2: rotary embedding, per-block summaries and product codes.
//
// One CTA per (token block j, sequence b, side): side 0 reads the block's bs
// tokens of q (all Hq heads), side 1 those of k (all Hkv heads), once, with
// 16-byte loads.  A warp takes one head at a time: lane (tg, c) rotates the
// 16-byte chunk c of both halves of its group of tokens, optionally writes
// the rotated values (the attention kernel reads them), and sums them in
// token order in float32; a fixed butterfly over the token groups then gives
// the block sum, scaled by 1/bs to the block mean.  The same warp then
// assigns the codes of the mean it just produced:
//   keys    : per subspace the codeword of largest <kbar_s, C[s,k]> (lowest
//             index on equal scores) -> product address sum_s c_s K^(P-1-s);
//   queries : per subspace the p codewords of largest score, best first.
// Pages: "Monodratic: a reproducible sparse attention mixer", section Mixer
// (routing acts on rotated keys and queries), and "Monodratic Claims Learned
// Routing Can Make Sparse Causal Attention More Selective", section
// "Monodratic Turns Sparse Attention Into a Retrieval Decision" (an address
// is a combination of several code choices).
//
// Rotary convention: coordinate i pairs with i + D/2; the pair at absolute
// position t turns by the float32 angle fp32(t) * omega_i, with omega_i =
// base^(-2i/D) rounded to float32 on the host; the block's (cos, sin) table
// is computed once per CTA with sincosf.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

constexpr int kSumThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSumThreads, 4)
summarize_kernel(const SummarizeArgs a) {
  using E = Elem<T>;
  constexpr int V = E::kVec;
  extern __shared__ float4 smem_f4[];
  const int j = blockIdx.x, b = blockIdx.y, side = blockIdx.z;
  if (!a.x[side]) return;
  const int bs = a.bs, D = a.D, half = D / 2;
  const int CH = half / V;                           // 16-byte chunks per half row
  const int TGW = 32 / CH;                           // token groups per warp
  const int per = bs / TGW;                          // tokens per lane
  const int H = a.H[side];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kSumThreads / 32;
  const int c = lane % CH, tg = lane / CH;

  float2* tab = reinterpret_cast<float2*>(smem_f4);  // [bs][half] (cos, sin)
  float* xbar_w = reinterpret_cast<float*>(tab + bs * half) + warp * D;   // this warp's summary

  // The key side pads this block's share of the posting lists with -1
  // (the list kernel, which runs next, only scatters).
  if (side == 1 && a.lists_fill) {
    const size_t share = (a.lists_per_seq + a.nb - 1) / a.nb;
    const size_t lo = static_cast<size_t>(j) * share;
    const size_t hi = lo + share < a.lists_per_seq ? lo + share : a.lists_per_seq;
    int32_t* l = a.lists_fill + static_cast<size_t>(b) * a.lists_per_seq;
    for (size_t e = lo + threadIdx.x; e < hi; e += kSumThreads) l[e] = -1;
  }

  // Rotation table of this block, computed once for every head.
  for (int e = threadIdx.x; e < bs * half; e += kSumThreads) {
    const int tt = e / half, i = e % half;
    const float ang = __fmul_rn(static_cast<float>(j * bs + tt), a.inv_freq[i]);
    float sn, cs;
    sincosf(ang, &sn, &cs);
    tab[e] = make_float2(cs, sn);
  }
  __syncthreads();

  const T* __restrict__ x = static_cast<const T*>(a.x[side]);
  T* __restrict__ xo = static_cast<T*>(a.xrot[side]);
  const size_t row = static_cast<size_t>(H) * D;     // elements per token
  const int dsub = D / a.P;
  const bool codes = side == 0 ? a.qcodes != nullptr : a.addr != nullptr;

  for (int h = warp; h < H; h += nwarps) {
    // Lane (tg, c) sums tokens tg*per .. tg*per+per-1 of chunk c, in order.
    const size_t base = (static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * bs + tg * per) * row +
                        static_cast<size_t>(h) * D + static_cast<size_t>(c) * V;
    float s1[V], s2[V];
#pragma unroll
    for (int v = 0; v < V; ++v) { s1[v] = 0.f; s2[v] = 0.f; }
    constexpr int kAhead = 2;                        // per is a power of two >= 2
    for (int t0 = 0; t0 < per; t0 += kAhead) {
      uint4 r1[kAhead], r2[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        const size_t off = base + static_cast<size_t>(t0 + u) * row;
        r1[u] = __ldg(reinterpret_cast<const uint4*>(x + off));
        r2[u] = __ldg(reinterpret_cast<const uint4*>(x + off + half));
      }
#pragma unroll
      for (int u = 0; u < kAhead; ++u) {
        float x1[V], x2[V], y1[V], y2[V];
        E::unpack(r1[u], x1);
        E::unpack(r2[u], x2);
        const float4* tr = reinterpret_cast<const float4*>(tab + (tg * per + t0 + u) * half + c * V);
#pragma unroll
        for (int v2 = 0; v2 < V / 2; ++v2) {
          const float4 cs = tr[v2];                  // (cos, sin) of two pairs
          const int v = 2 * v2;
          y1[v] = __fsub_rn(__fmul_rn(x1[v], cs.x), __fmul_rn(x2[v], cs.y));
          y2[v] = __fadd_rn(__fmul_rn(x2[v], cs.x), __fmul_rn(x1[v], cs.y));
          y1[v + 1] = __fsub_rn(__fmul_rn(x1[v + 1], cs.z), __fmul_rn(x2[v + 1], cs.w));
          y2[v + 1] = __fadd_rn(__fmul_rn(x2[v + 1], cs.z), __fmul_rn(x1[v + 1], cs.w));
          s1[v] = __fadd_rn(s1[v], y1[v]);
          s2[v] = __fadd_rn(s2[v], y2[v]);
          s1[v + 1] = __fadd_rn(s1[v + 1], y1[v + 1]);
          s2[v + 1] = __fadd_rn(s2[v + 1], y2[v + 1]);
        }
        if (xo) {
          const size_t off = base + static_cast<size_t>(t0 + u) * row;
          E::store(xo + off, y1);
          E::store(xo + off + half, y2);
        }
      }
    }
    // Combine the token groups: a fixed butterfly over the tg lane bits.
    for (int o = CH; o < 32; o <<= 1) {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        s1[v] = __fadd_rn(s1[v], __shfl_xor_sync(0xffffffffu, s1[v], o));
        s2[v] = __fadd_rn(s2[v], __shfl_xor_sync(0xffffffffu, s2[v], o));
      }
    }
    const float inv = 1.0f / static_cast<float>(bs);  // bs is a power of two
    if (tg == 0) {
      float* g = a.xbar[side] ? a.xbar[side] + ((static_cast<size_t>(b) * H + h) * a.nb + j) * D + c * V : nullptr;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const float m1 = s1[v] * inv, m2 = s2[v] * inv;
        xbar_w[c * V + v] = m1;
        xbar_w[half + c * V + v] = m2;
        if (g) { g[v] = m1; g[half + v] = m2; }
      }
    }
    __syncwarp();
    if (!codes) continue;

    // Codes of this head: lane scores codewords lane, lane+32, ... (K <= 128).
    int addr = 0;
    for (int sdx = 0; sdx < a.P; ++sdx) {
      float sc[4];
      int ki[4];
      const float4* xs4 = reinterpret_cast<const float4*>(xbar_w + sdx * dsub);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = lane + 32 * m;
        ki[m] = 0x7fffffff;
        sc[m] = -INFINITY;
        if (k < a.K) {
          const float4* cw = reinterpret_cast<const float4*>(a.codebooks + (static_cast<size_t>(sdx) * a.K + k) * dsub);
          float acc = 0.f;
          for (int d4 = 0; d4 < dsub / 4; ++d4) {
            const float4 xv = xs4[d4], cv = __ldg(cw + d4);
            acc = __fmaf_rn(xv.x, cv.x, acc);
            acc = __fmaf_rn(xv.y, cv.y, acc);
            acc = __fmaf_rn(xv.z, cv.z, acc);
            acc = __fmaf_rn(xv.w, cv.w, acc);
          }
          sc[m] = acc;
          ki[m] = k;
        }
      }
      const int rounds = side == 0 ? a.probes : 1;
      for (int rr = 0; rr < rounds; ++rr) {
        float bsc = sc[0];
        int bi = ki[0];
#pragma unroll
        for (int m = 1; m < 4; ++m)
          if (better(sc[m], ki[m], bsc, bi)) { bsc = sc[m]; bi = ki[m]; }
        warp_best(bsc, bi);
        if (side == 0) {
          if (lane == 0)
            a.qcodes[((((static_cast<size_t>(b) * H + h) * a.nb + j) * a.P + sdx) * a.probes) + rr] = bi;
#pragma unroll
          for (int m = 0; m < 4; ++m)
            if (ki[m] == bi) { sc[m] = -INFINITY; ki[m] = 0x7fffffff; }
        } else {
          addr = addr * a.K + bi;
        }
      }
    }
    if (side == 1 && lane == 0) a.addr[(static_cast<size_t>(b) * H + h) * a.nb + j] = addr;
    __syncwarp();
  }
}

size_t summarize_smem_bytes(int bs, int D, int Hq, int Hkv) {
  (void)Hq;
  (void)Hkv;
  return static_cast<size_t>(bs) * (D / 2) * sizeof(float2) + static_cast<size_t>(kSumThreads / 32) * D * sizeof(float);
}

cudaError_t launch_summarize(const SummarizeArgs& a, bool bf16, cudaStream_t st) {
  const dim3 grid(a.nb, a.B, 2);
  const size_t smem = summarize_smem_bytes(a.bs, a.D, a.H[0], a.H[1]);
  if (bf16) {
    auto k = summarize_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, kSumThreads, smem, st>>>(a);
  } else {
    auto k = summarize_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, kSumThreads, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mdr
