// K5 (CUDA cores): selected-set causal attention.
//
// For token t of query block j and query head hq: softmax over every token s
// of the blocks listed in sel[b,hq,j] with s <= t of scale * <q'_t, k'_s>,
// applied to v_s ("Monodratic: a reproducible sparse attention mixer",
// section Mixer: exact causal softmax over the selected set, with the
// selected values themselves, not a summary of them).
//
// One CTA per (b, hq, j); each warp owns query rows, lanes split the head
// dimension, and an online softmax (running max and sum, float32) folds the
// keys in one pass.  All arithmetic is float32, which is what the float32
// storage type needs: tf32 tensor-core products cannot meet a 1e-5 error.

#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace mdr {

template <typename T>
__global__ void __launch_bounds__(128)
attend_simt_kernel(const AttendArgs a) {
  __shared__ int32_t blocks[kMaxSel];
  __shared__ int nblk;
  grid_dependency_wait();
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;         // query blocks a.j0 .. a.j0 + nbr - 1
  const int bhq = blockIdx.x / nbr;
  const int j = a.j0 + static_cast<int>(blockIdx.x - bhq * nbr);
  const int hq = bhq % a.Hq;
  const int b = bhq / a.Hq;
  const int tile = bhq * a.nb + j;
  const int hkv = hq / (a.Hq / a.Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* q = static_cast<const T*>(a.q);
  const T* k = static_cast<const T*>(a.k);
  const T* v = static_cast<const T*>(a.v);
  T* out = static_cast<T*>(a.out);

  if (threadIdx.x == 0) {
    const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
    int n = 0;
    for (int e = 0; e < a.nsel; ++e) {
      const int id = row[e];
      if (id < 0) continue;
      if (id > j || id >= a.nb) { atomicExch(a.status, kDevBadSelection); continue; }
      blocks[n++] = id;
    }
    nblk = n;
  }
  __syncthreads();

  const int dm = a.D / 32;
  for (int r = warp; r < a.bs; r += blockDim.x / 32) {
    const int t = j * a.bs + r;
    float qv[4], acc[4];
    const size_t qoff = ((static_cast<size_t>(b) * a.S + t) * a.Hq + hq) * a.D;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      qv[m] = m < dm ? Elem<T>::to_float(q[qoff + lane + 32 * m]) : 0.f;
      acc[m] = 0.f;
    }
    float mx = -INFINITY, l = 0.f;
    for (int e = 0; e < nblk; ++e) {
      const int i = blocks[e];
      const int s_end = min((i + 1) * a.bs, t + 1);
      for (int s = i * a.bs; s < s_end; ++s) {
        const size_t koff = ((static_cast<size_t>(b) * a.S + s) * a.Hkv + hkv) * a.D;
        float dot = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m)
          if (m < dm) dot = __fmaf_rn(qv[m], Elem<T>::to_float(k[koff + lane + 32 * m]), dot);
        const float sc = warp_sum(dot) * a.scale;
        const float mnew = fmaxf(mx, sc);
        const float corr = expf(mx - mnew);
        const float p = expf(sc - mnew);
        l = l * corr + p;
#pragma unroll
        for (int m = 0; m < 4; ++m)
          if (m < dm) acc[m] = acc[m] * corr + p * Elem<T>::to_float(v[koff + lane + 32 * m]);
        mx = mnew;
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;   // nothing selected: zero output
    if (a.lse && lane == 0)
      a.lse[(static_cast<size_t>(b) * a.Hq + hq) * a.S + t] = l > 0.f ? mx + logf(l) : -INFINITY;
    const size_t ooff = ((static_cast<size_t>(b) * a.S + t) * a.Hq + hq) * a.D;
#pragma unroll
    for (int m = 0; m < 4; ++m)
      if (m < dm) {
        if constexpr (sizeof(T) == 4) out[ooff + lane + 32 * m] = acc[m] * inv;
        else out[ooff + lane + 32 * m] = __float2bfloat16_rn(acc[m] * inv);
      }
  }
}

cudaError_t launch_attend_simt(const AttendArgs& a, bool bf16, cudaStream_t st) {
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>(a.B) * a.Hq * nbr;
  const cudaError_t e = bf16 ? launch_pdl(attend_simt_kernel<__nv_bfloat16>, dim3(grid), dim3(128), 0, st, a)
                             : launch_pdl(attend_simt_kernel<float>, dim3(grid), dim3(128), 0, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
