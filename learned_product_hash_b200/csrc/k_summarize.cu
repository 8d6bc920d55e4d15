// K1 + K2: rotary embedding, per-block summaries and product codes.
//
// One CTA per (sequence b, token block j) reads the block's bs tokens of q
// (all Hq heads) and/or k (all Hkv heads) once with 16-byte loads, rotates
// them, optionally writes the rotated tensors (the attention kernel reads
// them), and reduces each head's rotated vectors to their block mean in
// float32.  It then assigns the codes of the means it just produced:
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
// base^(-2i/D) rounded to float32 on the host.  Block sums run over the
// tokens in ascending order, one float32 accumulator per coordinate.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

template <typename T>
__global__ void __launch_bounds__(128)
summarize_kernel(const SummarizeArgs a) {
  using E = Elem<T>;
  constexpr int V = E::kVec;
  extern __shared__ float4 smem_f4[];
  const int j = blockIdx.x, b = blockIdx.y;
  const int bs = a.bs, D = a.D, half = D / 2;
  const int chunks = half / V;                       // vectors per half row

  float2* tab = reinterpret_cast<float2*>(smem_f4);  // [bs][half] (cos, sin)
  float* xbar_s = reinterpret_cast<float*>(tab + bs * half);   // [Hq+Hkv][D]

  // Rotation table of this block: computed once, shared by every head.
  for (int e = threadIdx.x; e < bs * half; e += blockDim.x) {
    const int tt = e / half, i = e % half;
    const float ang = __fmul_rn(static_cast<float>(j * bs + tt), a.inv_freq[i]);
    float sn, cs;
    sincosf(ang, &sn, &cs);
    tab[e] = make_float2(cs, sn);
  }
  __syncthreads();

  const int items0 = a.x[0] ? a.H[0] * chunks : 0;
  const int items1 = a.x[1] ? a.H[1] * chunks : 0;
  for (int it = threadIdx.x; it < items0 + items1; it += blockDim.x) {
    const int side = it < items0 ? 0 : 1;
    const int r = side == 0 ? it : it - items0;
    const int H = a.H[side];
    const int h = r / chunks, c = r % chunks;
    const T* x = static_cast<const T*>(a.x[side]);
    T* xo = static_cast<T*>(a.xrot[side]);
    const size_t row = static_cast<size_t>(H) * D;            // elements per token
    const size_t base = (static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * bs) * row
                        + static_cast<size_t>(h) * D + static_cast<size_t>(c) * V;
    float s1[V], s2[V];
#pragma unroll
    for (int v = 0; v < V; ++v) { s1[v] = 0.f; s2[v] = 0.f; }
#pragma unroll 4
    for (int tt = 0; tt < bs; ++tt) {
      float x1[V], x2[V], y1[V], y2[V];
      const size_t off = base + static_cast<size_t>(tt) * row;
      E::load(x + off, x1);
      E::load(x + off + half, x2);
      const float2* tr = tab + tt * half + c * V;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        const float2 cssn = tr[v];
        y1[v] = __fsub_rn(__fmul_rn(x1[v], cssn.x), __fmul_rn(x2[v], cssn.y));
        y2[v] = __fadd_rn(__fmul_rn(x2[v], cssn.x), __fmul_rn(x1[v], cssn.y));
        s1[v] = __fadd_rn(s1[v], y1[v]);
        s2[v] = __fadd_rn(s2[v], y2[v]);
      }
      if (xo) {
        E::store(xo + off, y1);
        E::store(xo + off + half, y2);
      }
    }
    const float inv = 1.0f / static_cast<float>(bs);          // bs is a power of two
    float* xb = xbar_s + (side == 0 ? 0 : a.H[0]) * D + h * D + c * V;
#pragma unroll
    for (int v = 0; v < V; ++v) {
      xb[v] = s1[v] * inv;
      xb[half + v] = s2[v] * inv;
    }
    if (a.xbar[side]) {
      float* g = a.xbar[side] + ((static_cast<size_t>(b) * H + h) * a.nb + j) * D + c * V;
#pragma unroll
      for (int v = 0; v < V; ++v) {
        g[v] = s1[v] * inv;
        g[half + v] = s2[v] * inv;
      }
    }
  }
  __syncthreads();

  // Codes: one warp per (side, head).
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int dsub = D / a.P;
  const int nq = (a.x[0] && a.qcodes) ? a.H[0] : 0;
  const int nk = (a.x[1] && a.addr) ? a.H[1] : 0;
  for (int u = warp; u < nq + nk; u += nwarps) {
    const bool qside = u < nq;
    const int h = qside ? u : u - nq;
    const float* xb = xbar_s + (qside ? 0 : a.H[0]) * D + h * D;
    int addr = 0;
    for (int s = 0; s < a.P; ++s) {
      // Each lane scores codewords lane, lane+32, ... (K <= 128).
      float sc[4];
      int ki[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int k = lane + 32 * m;
        ki[m] = k;
        sc[m] = -INFINITY;
        if (k < a.K) {
          const float* cw = a.codebooks + (static_cast<size_t>(s) * a.K + k) * dsub;
          const float* xs = xb + s * dsub;
          float acc = 0.f;
          for (int d = 0; d < dsub; ++d) acc = __fmaf_rn(xs[d], __ldg(cw + d), acc);
          sc[m] = acc;
        } else {
          ki[m] = 0x7fffffff;
        }
      }
      const int rounds = qside ? a.probes : 1;
      for (int rr = 0; rr < rounds; ++rr) {
        float bsc = sc[0];
        int bi = ki[0];
#pragma unroll
        for (int m = 1; m < 4; ++m)
          if (better(sc[m], ki[m], bsc, bi)) { bsc = sc[m]; bi = ki[m]; }
        warp_best(bsc, bi);
        if (qside) {
          if (lane == 0)
            a.qcodes[((((static_cast<size_t>(b) * a.H[0] + h) * a.nb + j) * a.P + s) * a.probes) + rr] = bi;
#pragma unroll
          for (int m = 0; m < 4; ++m)
            if (ki[m] == bi) { sc[m] = -INFINITY; ki[m] = 0x7fffffff; }
        } else {
          addr = addr * a.K + bi;
        }
      }
    }
    if (!qside && lane == 0)
      a.addr[(static_cast<size_t>(b) * a.H[1] + h) * a.nb + j] = addr;
  }
}

size_t summarize_smem_bytes(int bs, int D, int Hq, int Hkv) {
  return static_cast<size_t>(bs) * (D / 2) * sizeof(float2) +
         static_cast<size_t>(Hq + Hkv) * D * sizeof(float);
}

cudaError_t launch_summarize(const SummarizeArgs& a, bool bf16, cudaStream_t st) {
  const dim3 grid(a.nb, a.B);
  const size_t smem = summarize_smem_bytes(a.bs, a.D, a.H[0], a.H[1]);
  if (bf16) {
    auto k = summarize_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, 128, smem, st>>>(a);
  } else {
    auto k = summarize_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    k<<<grid, 128, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace mdr
