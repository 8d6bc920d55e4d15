// Backward of the selected-set attention with the route held fixed: given
// dL/d(out), dL/dq, dL/dk, dL/dv through the causal softmax over the tokens
// of the selected blocks and through the rotary embedding.  "Monodratic
// Claims Learned Routing Can Make Sparse Causal Attention More Selective",
// section "The 99.35 Percent Result Does Not Establish Language Quality":
// hard top-k choices pass no ordinary gradient through the chosen index, so
// nothing flows to the codebooks or the block summaries.
//
// The CUDA-core path (float32 storage; bf16 storage runs on the tensor cores
// in k_backward_tc.cu).  Four kernels, float32 arithmetic, every floating-point sum in a fixed
// order (the only atomics count list entries in shared memory, whose integer
// totals do not depend on order), so a call is deterministic:
//   bwd_rotate_kernel  float32 rotated copies q', k' (the angle of the
//                      forward: the float32 product t * omega_i, sincosf).
//   bwd_rev_kernel     one CTA per (sequence, KV head): for every key block,
//                      the (query head, query block) pairs whose selection
//                      holds it, in (head, block, slot) order -- a stable
//                      counting sort of the selection (counts, prefix sums,
//                      then rounds of 32 entries per warp: ranks within a
//                      warp by __match_any_sync, each warp's starting rank
//                      per key block by a prefix over a [warps][nb] count
//                      table; one warp walks the entries when the table does
//                      not fit in shared memory).
//   bwd_dq_kernel      one or more CTAs per (sequence, query head, query
//                      block), thread = (query token, 16 coordinates):
//                      pass 1 over the selected blocks (K, V staged in shared
//                      memory) recomputes the row maximum, sum and output ->
//                      log-sum-exp and D_t = dO_t . O_t; pass 2 recomputes
//                      P = exp(s - lse), dS = P (dO.v - D_t), dq' += scale dS k';
//                      dq = R(t)^T dq'.
//   bwd_dkdv_kernel    one or more CTAs per (sequence, KV head, key block),
//                      thread = (key token, 16 coordinates): walks the
//                      block's reverse list,
//                      staging each query block's q', dO, lse, D, and adds
//                      dv += P dO, dk' += scale dS q' (t >= s only);
//                      dk = R(s)^T dk'.
// No thread waits on another block or on a flag: nothing here can hang.

#include <cmath>

#include "common.cuh"
#include "kernels.h"

namespace mdr {

namespace {

__device__ __forceinline__ float ld_f(const float* p, long long i) { return p[i]; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }

}  // namespace

template <typename T>
__global__ void bwd_rotate_kernel(const BwdArgs a) {
  __shared__ float om[64];
  if (threadIdx.x < a.D / 2) om[threadIdx.x] = a.inv_freq[threadIdx.x];
  __syncthreads();
  grid_dependency_wait();                          // q, k may come from the previous kernel
  const int half = a.D / 2;
  const long long nq = static_cast<long long>(a.B) * a.S * a.Hq * half;
  const long long nk = static_cast<long long>(a.B) * a.S * a.Hkv * half;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long e = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; e < nq + nk; e += stride) {
    const bool isq = e < nq;
    const long long f = isq ? e : e - nq;
    const int H = isq ? a.Hq : a.Hkv;
    const int i = static_cast<int>(f % half);
    const long long row = f / half;                          // (b * S + t) * H + h
    const int t = static_cast<int>((row / H) % a.S);
    const T* x = static_cast<const T*>(isq ? a.q : a.k);
    float* y = isq ? a.qr : a.kr;
    float sn, cs;
    sincosf(static_cast<float>(t) * om[i], &sn, &cs);
    const float x1 = ld_f(x, row * a.D + i), x2 = ld_f(x, row * a.D + i + half);
    y[row * a.D + i] = x1 * cs - x2 * sn;
    y[row * a.D + i + half] = x2 * cs + x1 * sn;
  }
}

constexpr int kRevThreads = 512;

__global__ void __launch_bounds__(kRevThreads) bwd_rev_kernel(const BwdArgs a, const int nw) {
  extern __shared__ int rsm[];
  int* cnt = rsm;                                  // [nb]
  int* off = rsm + a.nb;                           // [nb + 1]
  int* cw = off + a.nb + 1;                        // [nw][nb] when nw > 0
  const int b = blockIdx.x / a.Hkv, h = blockIdx.x % a.Hkv;
  const int g = a.Hq / a.Hkv;
  const int E = g * a.nb * a.nsel;                 // entries (hl, j, slot); < 2^31 (checked on the host)
  const int32_t* sel0 = a.sel + (static_cast<long long>(b) * a.Hq + static_cast<long long>(h) * g) * a.nb * a.nsel;
  const int tid = threadIdx.x;
  for (int i = tid; i < a.nb; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  grid_dependency_wait();                          // sel may come from the previous kernel
  // Counts (order-free).
  for (int e = tid; e < E; e += blockDim.x) {
    const int j = (e / a.nsel) % a.nb;
    const int id = sel0[e];
    if (id >= 0 && id <= j) atomicAdd(&cnt[id], 1);
  }
  __syncthreads();
  // Exclusive prefix sums by warp 0, 32 blocks at a time.
  const int warp = tid >> 5, lane = tid & 31;
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < a.nb; base += 32) {
      const int i = base + lane;
      const int c = i < a.nb ? cnt[i] : 0;
      int x = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (i < a.nb) off[i] = run + x - c;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) off[a.nb] = run;
  }
  __syncthreads();
  int32_t* roff = a.rev_off + static_cast<long long>(blockIdx.x) * (a.nb + 1);
  for (int i = tid; i <= a.nb; i += blockDim.x) roff[i] = off[i];
  for (int i = tid; i < a.nb; i += blockDim.x) cnt[i] = 0;   // reused as running counts
  __syncthreads();
  int32_t* rev = a.rev + static_cast<long long>(blockIdx.x) * E;
  const int per_head = a.nsel * a.nb;
  if (nw > 0) {
    // Stable placement in rounds of nw * 32 entries: (1) ranks within each
    // warp's 32 consecutive entries, the lowest peer recording its group's
    // size in the warp's row of the table; (2) per key block, a prefix over
    // the warps gives each warp's starting rank and advances the running
    // count; (3) each entry lands at its block's offset + starting rank +
    // rank within the warp.
    const unsigned lower = (1u << lane) - 1u;
    for (int r0 = 0; r0 < E; r0 += nw * 32) {
      for (int x = tid; x < nw * a.nb; x += blockDim.x) cw[x] = 0;
      __syncthreads();
      const int e = r0 + warp * 32 + lane;
      int id = -1, code = 0;
      if (warp < nw && e < E) {
        const int hl = e / per_head, j = (e - hl * per_head) / a.nsel;
        const int v = sel0[e];
        if (v >= 0 && v <= j) {
          id = v;
          code = hl * a.nb + j;
        }
      }
      int rk = 0;
      if (warp < nw) {
        const unsigned vm = __ballot_sync(0xffffffffu, id >= 0);
        if (id >= 0) {
          const unsigned peers = __match_any_sync(vm, id);
          rk = __popc(peers & lower);
          if (rk == 0) cw[warp * a.nb + id] = __popc(peers);
        }
      }
      __syncthreads();
      for (int x = tid; x < a.nb; x += blockDim.x) {
        int run = cnt[x];
        for (int w = 0; w < nw; ++w) {
          const int t = cw[w * a.nb + x];
          cw[w * a.nb + x] = run;
          run += t;
        }
        cnt[x] = run;
      }
      __syncthreads();
      if (id >= 0) rev[off[id] + cw[warp * a.nb + id] + rk] = code;
      __syncthreads();                             // the table is cleared for the next round
    }
  } else if (warp == 0) {
    // One warp walks the entries 32 at a time; the selection is read four
    // steps ahead so the loads overlap.
    int ahead[4];
    for (int base = 0; base < E; base += 32) {
      const int u = (base >> 5) & 3;
      if (u == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = base + 32 * q + lane;
          ahead[q] = e < E ? sel0[e] : -1;
        }
      }
      int loaded = ahead[0];
#pragma unroll
      for (int q = 1; q < 4; ++q)
        if (q == u) loaded = ahead[q];
      const int e = base + lane;
      int id = -1, j = 0, hl = 0;
      if (e < E) {
        hl = e / per_head;
        j = (e - hl * per_head) / a.nsel;
        id = loaded;
        if (id > j) id = -1;
      }
      const bool ok = id >= 0;
      const unsigned peers = __match_any_sync(0xffffffffu, ok ? id : -1 - lane);
      if (ok) {
        const int rank = cnt[id] + __popc(peers & ((1u << lane) - 1u));
        rev[off[id] + rank] = hl * a.nb + j;
      }
      __syncwarp();
      if (ok && (peers & ((1u << lane) - 1u)) == 0) cnt[id] += __popc(peers);
      __syncwarp();
    }
  }
}

// Threads of one token: PARTS = D / 16, each holding 16 coordinates; a CTA
// of at most 256 threads covers tpc = min(bs, 256 / PARTS) tokens, so a
// block of bs tokens takes bs / tpc CTAs.
template <int PARTS>
__device__ __forceinline__ float part_sum(float v) {
#pragma unroll
  for (int o = 1; o < PARTS; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kC = 16;             // coordinates per thread

template <typename T, int PARTS>
__global__ void __launch_bounds__(256, 1) bwd_dq_kernel(const BwdArgs a) {
  extern __shared__ float qsm[];
  const int bs = a.bs, D = a.D;                    // D == PARTS * kC
  const int tpc = blockDim.x / PARTS, pieces = bs / tpc;
  float* Ks = qsm;                                 // [bs][D]
  float* Vs = qsm + bs * D;                        // [bs][D]
  const int tl = threadIdx.x / PARTS, part = threadIdx.x % PARTS;
  const long long route = blockIdx.x / pieces;     // (b * Hq + hq) * nb + j
  const int tq = static_cast<int>(blockIdx.x % pieces) * tpc + tl;   // token within the query block
  const int tq_warp_last = static_cast<int>(blockIdx.x % pieces) * tpc + ((threadIdx.x | 31) / PARTS);
  const int j = static_cast<int>(route % a.nb);
  const int hq = static_cast<int>((route / a.nb) % a.Hq);
  const int b = static_cast<int>(route / (static_cast<long long>(a.nb) * a.Hq));
  const int h = hq / (a.Hq / a.Hkv);
  const int t = j * bs + tq;
  const long long qrow = (static_cast<long long>(b) * a.S + t) * a.Hq + hq;
  const T* dout = static_cast<const T*>(a.dout);
  const T* vin = static_cast<const T*>(a.v);
  grid_dependency_wait();                          // the rotated copies come from the previous kernels
  float qv[kC], dov[kC], acc[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    qv[c] = a.qr[qrow * D + part * kC + c];
    dov[c] = ld_f(dout, qrow * D + part * kC + c);
    acc[c] = 0.f;
  }
  const int32_t* row = a.sel + route * a.nsel;
  float m = -INFINITY, l = 0.f, lse = 0.f, delta = 0.f;
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 1) {
      // Row statistics of pass 0; a row with no visible key keeps dq = 0.
      float o_dot = 0.f;
#pragma unroll
      for (int c = 0; c < kC; ++c) o_dot = __fmaf_rn(dov[c], l > 0.f ? acc[c] / l : 0.f, o_dot);
      delta = part_sum<PARTS>(o_dot);
      lse = l > 0.f ? m + logf(l) : INFINITY;
      if (part == 0) {
        const long long si = (static_cast<long long>(b) * a.Hq + hq) * a.S + t;
        a.lse[si] = lse;
        a.delta[si] = delta;
      }
#pragma unroll
      for (int c = 0; c < kC; ++c) acc[c] = 0.f;
    }
    for (int slot = 0; slot < a.nsel; ++slot) {
      const int blk = row[slot];
      if (blk < 0 || blk > j) {
        if (pass == 0 && blk > j && threadIdx.x == 0 && a.status) atomicExch(a.status, 2);
        continue;
      }
      __syncthreads();                             // the previous block's tiles are no longer read
      for (int e = threadIdx.x; e < bs * D; e += blockDim.x) {
        const int s = e / D, d = e - s * D;
        const long long krow = (static_cast<long long>(b) * a.S + blk * bs + s) * a.Hkv + h;
        Ks[e] = a.kr[krow * D + d];
        Vs[e] = ld_f(vin, krow * D + d);
      }
      __syncthreads();
      // Keys s <= t.  The loop runs to the warp's last token (the sums over a
      // token's threads need every lane) and masks later keys.
      const int last = blk == j ? (tq_warp_last < bs - 1 ? tq_warp_last : bs - 1) : bs - 1;
      for (int s = 0; s <= last; ++s) {
        const bool vis = blk != j || s <= tq;
        const float* kp = Ks + s * D + part * kC;
        const float* vp = Vs + s * D + part * kC;
        float dot = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < kC; ++c) dot = __fmaf_rn(qv[c], kp[c], dot);
        if (pass == 1) {
#pragma unroll
          for (int c = 0; c < kC; ++c) dp = __fmaf_rn(dov[c], vp[c], dp);
          dp = part_sum<PARTS>(dp);
        }
        const float sc = a.scale * part_sum<PARTS>(dot);
        if (!vis) continue;
        if (pass == 0) {
          if (sc > m) {                            // online softmax: rescale the running sums
            const float r = expf(m - sc);
            l *= r;
#pragma unroll
            for (int c = 0; c < kC; ++c) acc[c] *= r;
            m = sc;
          }
          const float p = expf(sc - m);
          l += p;
#pragma unroll
          for (int c = 0; c < kC; ++c) acc[c] = __fmaf_rn(p, vp[c], acc[c]);
        } else {
          const float ds = expf(sc - lse) * (dp - delta);
#pragma unroll
          for (int c = 0; c < kC; ++c) acc[c] = __fmaf_rn(a.scale * ds, kp[c], acc[c]);
        }
      }
    }
  }
  // dq = R(t)^T dq': coordinate i pairs with i + D/2, held by part ^ (PARTS/2).
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const float other = __shfl_xor_sync(0xffffffffu, acc[c], PARTS / 2);
    float sn, cs;
    sincosf(static_cast<float>(t) * a.inv_freq[(part * kC + c) % (D / 2)], &sn, &cs);
    a.dq[qrow * D + part * kC + c] = part < PARTS / 2 ? acc[c] * cs + other * sn    // y1 c + y2 s
                                                      : acc[c] * cs - other * sn;   // y2 c - y1 s
  }
}

template <typename T, int PARTS>
__global__ void __launch_bounds__(256, 1) bwd_dkdv_kernel(const BwdArgs a) {
  extern __shared__ float ksm[];
  const int bs = a.bs, D = a.D;
  const int tpc = blockDim.x / PARTS, pieces = bs / tpc;
  float* Qs = ksm;                                 // [bs][D]
  float* Os = ksm + bs * D;                        // [bs][D] upstream gradient
  float* Ls = ksm + 2 * bs * D;                    // [bs] lse
  float* Ds = Ls + bs;                             // [bs] delta
  const int tl = threadIdx.x / PARTS, part = threadIdx.x % PARTS;
  const long long kb = blockIdx.x / pieces;        // (b * Hkv + h) * nb + i
  const int ts = static_cast<int>(blockIdx.x % pieces) * tpc + tl;            // key token within the block
  const int ts_warp_first = static_cast<int>(blockIdx.x % pieces) * tpc + ((threadIdx.x & ~31u) / PARTS);
  const int i = static_cast<int>(kb % a.nb);
  const long long bh = kb / a.nb;
  const int h = static_cast<int>(bh % a.Hkv);
  const int b = static_cast<int>(bh / a.Hkv);
  const int g = a.Hq / a.Hkv;
  const int s = i * bs + ts;
  const long long krow = (static_cast<long long>(b) * a.S + s) * a.Hkv + h;
  const T* dout = static_cast<const T*>(a.dout);
  const T* vin = static_cast<const T*>(a.v);
  grid_dependency_wait();                          // lse, delta and the reverse index come from the previous kernels
  float kv[kC], vv[kC], dk[kC], dv[kC];
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    kv[c] = a.kr[krow * D + part * kC + c];
    vv[c] = ld_f(vin, krow * D + part * kC + c);
    dk[c] = 0.f;
    dv[c] = 0.f;
  }
  const int32_t* roff = a.rev_off + bh * (a.nb + 1);
  const int32_t* rev = a.rev + bh * (static_cast<long long>(g) * a.nb * a.nsel);
  const int e0 = roff[i], e1 = roff[i + 1];
  for (int e = e0; e < e1; ++e) {
    const int code = rev[e];
    const int hl = code / a.nb, j = code - hl * a.nb;
    const int hq = h * g + hl;
    __syncthreads();                               // the previous query block's tiles are no longer read
    for (int x = threadIdx.x; x < bs * D; x += blockDim.x) {
      const int tt = x / D, d = x - tt * D;
      const long long qrow = (static_cast<long long>(b) * a.S + j * bs + tt) * a.Hq + hq;
      Qs[x] = a.qr[qrow * D + d];
      Os[x] = ld_f(dout, qrow * D + d);
    }
    for (int tt = threadIdx.x; tt < bs; tt += blockDim.x) {
      const long long si = (static_cast<long long>(b) * a.Hq + hq) * a.S + j * bs + tt;
      Ls[tt] = a.lse[si];
      Ds[tt] = a.delta[si];
    }
    __syncthreads();
    // Queries t >= s.  The loop starts at the warp's first key token (the
    // sums over a token's threads need every lane) and masks earlier queries.
    const int first = j == i ? ts_warp_first : 0;
    for (int tt = first; tt < bs; ++tt) {
      const bool vis = j != i || tt >= ts;
      const float* qp = Qs + tt * D + part * kC;
      const float* op = Os + tt * D + part * kC;
      float dot = 0.f, dp = 0.f;
#pragma unroll
      for (int c = 0; c < kC; ++c) { dot = __fmaf_rn(kv[c], qp[c], dot); dp = __fmaf_rn(vv[c], op[c], dp); }
      const float sdot = part_sum<PARTS>(dot), sdp = part_sum<PARTS>(dp);
      if (!vis) continue;
      const float p = expf(a.scale * sdot - Ls[tt]);
      const float ds = p * (sdp - Ds[tt]);
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        dv[c] = __fmaf_rn(p, op[c], dv[c]);
        dk[c] = __fmaf_rn(a.scale * ds, qp[c], dk[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < kC; ++c) {
    const float other = __shfl_xor_sync(0xffffffffu, dk[c], PARTS / 2);
    float sn, cs;
    sincosf(static_cast<float>(s) * a.inv_freq[(part * kC + c) % (D / 2)], &sn, &cs);
    a.dk[krow * D + part * kC + c] = part < PARTS / 2 ? dk[c] * cs + other * sn : dk[c] * cs - other * sn;
    a.dv[krow * D + part * kC + c] = dv[c];
  }
}

size_t bwd_rev_smem(int nb) { return static_cast<size_t>(2 * nb + 1) * sizeof(int); }

template <typename T, int PARTS>
static cudaError_t launch_grad_kernels(const BwdArgs& a, cudaStream_t st) {
  const int tpc = a.bs < 256 / PARTS ? a.bs : 256 / PARTS;
  const long long pieces = a.bs / tpc;
  cudaError_t e;
  {
    const size_t smem = static_cast<size_t>(2) * a.bs * a.D * sizeof(float);
    const auto k = bwd_dq_kernel<T, PARTS>;
    e = cached_allow_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(k, dim3(static_cast<unsigned>(static_cast<long long>(a.B) * a.Hq * a.nb * pieces)),
                   dim3(tpc * PARTS), smem, st, a);
    if (e != cudaSuccess) return e;
  }
  {
    const size_t smem = (static_cast<size_t>(2) * a.bs * a.D + 2 * a.bs) * sizeof(float);
    const auto k = bwd_dkdv_kernel<T, PARTS>;
    e = cached_allow_smem(reinterpret_cast<const void*>(k), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(k, dim3(static_cast<unsigned>(static_cast<long long>(a.B) * a.Hkv * a.nb * pieces)),
                   dim3(tpc * PARTS), smem, st, a);
  }
  return e;
}

template <typename T>
static cudaError_t launch_grad_for(const BwdArgs& a, cudaStream_t st) {
  switch (a.D) {
    case 32: return launch_grad_kernels<T, 2>(a, st);
    case 64: return launch_grad_kernels<T, 4>(a, st);
    case 128: return launch_grad_kernels<T, 8>(a, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_bwd_rev(const BwdArgs& a, cudaStream_t st) {
  // As many warp rows of the placement table as fit beside the counts and
  // offsets (none: one warp walks the entries).
  constexpr int kSmemInts = 227 * 1024 / 4 - 64;
  const long long base_ints = 2LL * a.nb + 1;
  long long nw = a.nb > 0 ? (kSmemInts - base_ints) / a.nb : 0;
  nw = nw < kRevThreads / 32 ? nw : kRevThreads / 32;
  if (nw < 2) nw = 0;
  const size_t smem = bwd_rev_smem(a.nb) + static_cast<size_t>(nw) * a.nb * sizeof(int);
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(bwd_rev_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(bwd_rev_kernel, dim3(a.B * a.Hkv), dim3(kRevThreads), smem, st, a, static_cast<int>(nw));
}

cudaError_t launch_backward(const BwdArgs& a, bool bf16, cudaStream_t st) {
  if (a.D != 32 && a.D != 64 && a.D != 128) return cudaErrorInvalidValue;
  const int sms = cached_sm_count();
  if (sms <= 0) return cudaErrorUnknown;
  cudaError_t e;
  {
    const auto k = bf16 ? bwd_rotate_kernel<__nv_bfloat16> : bwd_rotate_kernel<float>;
    e = launch_pdl(k, dim3(sms * 4), dim3(256), 0, st, a);
    if (e != cudaSuccess) return e;
  }
  e = launch_bwd_rev(a, st);
  if (e != cudaSuccess) return e;
  e = bf16 ? launch_grad_for<__nv_bfloat16>(a, st) : launch_grad_for<float>(a, st);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
