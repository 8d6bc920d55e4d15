// Backward of the selected-set attention on the tensor cores (bf16 storage):
// dL/dq, dL/dk, dL/dv for dL/d(out), the route held fixed.  "Monodratic
// Claims Learned Routing Can Make Sparse Causal Attention More Selective",
// section "The 99.35 Percent Result Does Not Establish Language Quality":
// hard top-k choices pass no ordinary gradient through the chosen index, so
// the gradient is that of the causal softmax over the selected tokens and of
// the rotary embedding; nothing reaches the codebooks or the summaries.
//
// Inputs are the rotated copies q', k' (bf16, written by the summary kernel
// exactly as for the forward), v and the upstream gradient dO, all read as
// 128-byte-swizzled [bs x 64] boxes by TMA; every product runs as a
// tcgen05.mma (bf16 operands, float32 accumulators in tensor memory).  Scores
// are kept in log2 units (scale * log2(e) folded in), exponentials are
// ex2.approx.
//
//   bwd_dq_tc_kernel    one query tile (b, hq, j) at a time, persistent.
//     pass 1, per selected block: S = Q K^T; the running maximum and sum of
//       each row; P = 2^(S - max) (bf16) into shared memory; O += P V.  At
//       the end: lse = max + log2(sum) and Delta = <dO, O> / sum per row,
//       stored for the key-side kernel.
//     pass 2, per selected block: S = Q K^T and dP = dO V^T; P = 2^(S - lse),
//       dS = P (dP - Delta) (bf16) into shared memory; dQ += dS K (K read
//       MN-major from its TMA tile).  Epilogue: dq = R(t)^T (scale dQ).
//   bwd_dkdv_ws_kernel  one key block (b, hkv, i) at a time, persistent, over
//     the block's reverse list (the (query head, query block) pairs that
//     selected it, in a fixed order): S^T = K Q^T and dP^T = V dO^T;
//     P^T = 2^(S^T - lse_t), dS^T = P^T (dP^T - Delta_t) (bf16); dV += P^T dO,
//     dK += dS^T Q.  Epilogue: dv = dV, dk = R(s)^T (scale dK).  Warp-
//     specialised (see the kernel).
// The causal mask applies where the key block is the query block (key s >
// query t is masked).  Warp w of the four that read accumulators owns TMEM
// subpartition w (rows 16w..16w+15 for bs = 64, two threads per row
// splitting the columns; rows 32w..32w+31 for bs = 128).  In the dq kernel
// thread 0 issues the TMA loads and the MMAs and the next blocks' tiles load
// into a ring of slots while the current one is computed; the dk/dv kernel
// has a TMA warp and an MMA warp of its own.  Sums run in a fixed order and there
// are no atomics, so a call is deterministic.  Every wait is bounded (2 s of
// wall time): a wait that runs out writes status 1, the CTA waits (bounded)
// for its own copies and MMAs, frees its tensor memory and returns.

#include <cuda.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace mdr {

namespace {

constexpr uint64_t kBwWaitNs = 2000000000ull;
constexpr uint64_t kBwBudgetNs = 10000000000ull;  // a CTA gives up after 10 s of wall time in total
constexpr int kBwThreads = 128;

// Where a CTA gave up, recorded (first one wins) in the second status word:
// 100 * kernel (1 dq, 2 dk/dv) + site, plus 50 when the CTA's time budget ran
// out rather than the wait itself; site 90+ are index checks that failed.
enum BwSite : int {
  kSiteQ = 1, kSiteKV = 2, kSiteS = 3, kSiteMM = 4, kSiteEntry = 5,
  kSiteRevRange = 90, kSiteRevCode = 91,
};

__device__ __forceinline__ void record_site(int32_t* status, int code) {
  atomicCAS(status + 1, 0, code);
}

constexpr int pow2_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

template <int BS, int D>
struct BwCfg {
  static constexpr bool kHR = (BS == 64);            // rows in lanes 0-15: two threads per row
  static constexpr int kTile = BS * D * 2;           // bf16 [BS x D]: D/64 regions
  static constexpr int kRegion = BS * 128;           // one 64-column region of a [BS x *] tile
  static constexpr int kPTile = BS * BS * 2;         // bf16 [BS x BS]: BS/64 regions
  static constexpr int kCtl = 1024;                  // barriers, omega, ids, misc
  // dq kernel: Q, dO, NKV (K, V) slots, P / dS.  The slots hold the next
  // blocks' tiles in flight while the current one computes.  At bs = 64 the
  // kernel needs 256 TMEM columns, so two CTAs share an SM (their phases
  // overlap); shared memory is sized for that.  At bs = 128 one CTA holds
  // all 512 columns and takes deeper rings instead.
  static constexpr int NKV = (BS == 64) ? (D == 64 ? 5 : 2) : (D == 128 ? 2 : 5);
  static constexpr int qOffQ = 0;
  static constexpr int qOffO = kTile;
  static constexpr int qOffKV = 2 * kTile;
  static constexpr int qOffP = qOffKV + NKV * 2 * kTile;
  static constexpr int qOffCtl = qOffP + kPTile;
  static constexpr int qSmem = qOffCtl + kCtl;
  static constexpr int qCols = pow2_cols(2 * BS + D);
  static constexpr int qColS = 0, qColP = BS, qColO = 2 * BS;
  // dk/dv kernel: an entry slot holds a query tile's Q, dO, lse and Delta, and a header (its query block)
  static constexpr int kSlot = (2 * kTile + 2 * BS * 4 + 16 + 1023) / 1024 * 1024;   // + a 16-byte header
  static_assert(qSmem <= 232448, "shared memory per CTA");
  static_assert(kTile % 1024 == 0 && kPTile % 1024 == 0, "1024-byte aligned tiles");
  // D-column geometry of a thread: W columns at lo and W at D/2 + lo, NP times.
  static constexpr int W = kHR ? D / 4 : 32;
  static constexpr int NP = kHR ? 1 : D / 64;
  // score-column geometry: NC chunks of 32 columns
  static constexpr int NC = kHR ? 1 : BS / 32;
};

// Control block at the end of shared memory.
struct Ctl {
  uint64_t bar[16];
  float om[64];
  int16_t ids[64];
  uint32_t tmem;
  int nblk;
  int abort;
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// K-major operand descriptor of a [rows x D] tile (D/64 regions) at K step kk.
template <int BS>
__device__ __forceinline__ uint64_t kmaj(uint32_t s, int kk) {
  return tc::smem_desc_sw128(s, 16, 1024) + static_cast<uint64_t>(((kk / 4) * (BS * 128) + (kk % 4) * 32) / 16);
}
// MN-major operand descriptor (N = D in 64-column regions) at K step kk (16 rows).
template <int BS>
__device__ __forceinline__ uint64_t mnmaj(uint32_t s, int kk) {
  return tc::smem_desc_sw128(s, BS * 128, 1024) + static_cast<uint64_t>(kk * 128);
}

// Thread geometry over the accumulator rows.
template <int BS, int D>
struct Rows {
  using C = BwCfg<BS, D>;
  int warp, lane, r, tsub;
  uint32_t lane_base;
  __device__ Rows() {
    warp = threadIdx.x >> 5;
    lane = threadIdx.x & 31;
    const int sp = warp & 3;                         // TMEM subpartition of this warp
    tsub = C::kHR ? (lane >> 4) : 0;
    r = C::kHR ? sp * 16 + (lane & 15) : sp * 32 + lane;
    lane_base = static_cast<uint32_t>(sp * 32) << 16;
  }
  // 32 score columns of chunk c (first column returned); all lanes take part.
  __device__ __forceinline__ int ld_scores(uint32_t tcol, int c, float* v) const {
    if constexpr (C::kHR) {
      tc::tmem_ld16x2_32(tcol + lane_base, v);
      return 32 * tsub;
    } else {
      tc::tmem_ld32(tcol + 32 * c + lane_base, v);
      return 32 * c;
    }
  }
  // W D-columns at offset off (0 or D/2, plus the pair's chunk) of part pp.
  __device__ __forceinline__ void ld_d(uint32_t tcol, int pp, int half, float* v) const {
    const uint32_t at = tcol + (half ? D / 2 : 0) + (C::kHR ? 0 : 32 * pp) + lane_base;
    if constexpr (C::kHR && D == 64) tc::tmem_ld16x2_16(at, v);
    else if constexpr (C::kHR) tc::tmem_ld16x2_32(at, v);
    else tc::tmem_ld32(at, v);
  }
  __device__ __forceinline__ void st_d(uint32_t tcol, int pp, int half, const float* v) const {
    const uint32_t at = tcol + (half ? D / 2 : 0) + (C::kHR ? 0 : 32 * pp) + lane_base;
    if constexpr (C::kHR && D == 64) tc::tmem_st16x2_16(at, v);
    else if constexpr (C::kHR) tc::tmem_st16x2_32(at, v);
    else tc::tmem_st32(at, v);
  }
  // First D-column of the lower half held for part pp.
  __device__ __forceinline__ int col_lo(int pp) const { return C::kHR ? C::W * tsub : 32 * pp; }
  // Sum of a per-thread partial over the row's threads.
  __device__ __forceinline__ float row_sum(float x) const {
    if constexpr (C::kHR) x += __shfl_xor_sync(0xffffffffu, x, 16);
    return x;
  }
  __device__ __forceinline__ float row_max(float x) const {
    if constexpr (C::kHR) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
    return x;
  }
};

// Eight bf16 values of row r at columns c0..c0+7 (c0 % 8 == 0) of a
// K-major, 128-byte-swizzled [BS x *] tile.
template <int BS>
__device__ __forceinline__ void st_bf16x8(uint8_t* tile, int r, int c0, const float* x) {
  const int chunk = ((c0 % 64) / 8) ^ (r & 7);
  *reinterpret_cast<uint4*>(tile + (c0 / 64) * (BS * 128) + r * 128 + chunk * 16) =
      make_uint4(pack2(x[0], x[1]), pack2(x[2], x[3]), pack2(x[4], x[5]), pack2(x[6], x[7]));
}

// Dot product of W float32 values with W bf16 values in global memory.
template <int W>
__device__ __forceinline__ float dot_bf16(const float* x, const __nv_bfloat16* g) {
  float s = 0.f;
#pragma unroll
  for (int q = 0; q < W / 8; ++q) {
    float y[8];
    Elem<__nv_bfloat16>::load(g + 8 * q, y);
#pragma unroll
    for (int e = 0; e < 8; ++e) s = __fmaf_rn(x[8 * q + e], y[e], s);
  }
  return s;
}

// y = R(t)^T (scale * x) for the pair (lo, hi) = coordinates (i, i + D/2),
// i = i0 .. i0 + W - 1, written as float32 to row out at columns i and i + D/2.
template <int W, int D>
__device__ __forceinline__ void rotate_store(const float* lo, const float* hi, int i0, int t, float scale,
                                             const float* om, float* out) {
#pragma unroll
  for (int q = 0; q < W / 4; ++q) {
    float a[4], b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int i = i0 + 4 * q + e;
      float sn, cs;
      sincosf(static_cast<float>(t) * om[i], &sn, &cs);
      const float y1 = scale * lo[4 * q + e], y2 = scale * hi[4 * q + e];
      a[e] = y1 * cs + y2 * sn;
      b[e] = y2 * cs - y1 * sn;
    }
    *reinterpret_cast<float4*>(out + i0 + 4 * q) = make_float4(a[0], a[1], a[2], a[3]);
    *reinterpret_cast<float4*>(out + D / 2 + i0 + 4 * q) = make_float4(b[0], b[1], b[2], b[3]);
  }
}

template <int W>
__device__ __forceinline__ void store_f32(float* out, const float* x) {
#pragma unroll
  for (int q = 0; q < W / 4; ++q)
    *reinterpret_cast<float4*>(out + 4 * q) = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
}

}  // namespace

// ---------------------------------------------------------------- dq kernel
template <int BS, int D>
__global__ void __launch_bounds__(kBwThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                 const BwdArgs a) {
  using C = BwCfg<BS, D>;
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(a.status, kDevMisaligned);
    return;
  }
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + C::qOffCtl);
  const uint32_t base = smem_u32(smem);
  const uint32_t sQ = base + C::qOffQ, sO = base + C::qOffO, sKV = base + C::qOffKV, sP = base + C::qOffP;
  uint8_t* pP = smem + C::qOffP;
  enum { bQ = 0, bS = 1, bMM = 2, bFin = 3, bKV0 = 4 };     // bKV0 .. bKV0 + NKV - 1
  static_assert(bKV0 + C::NKV <= 16, "barrier space");
  auto BAR = [&](int i) { return smem_u32(&ctl.bar[i]); };
  const Rows<BS, D> R;
  if (R.warp == 0) {
    tmem_alloc(smem_u32(&ctl.tmem), C::qCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < bKV0 + C::NKV; ++i) mbar_init(BAR(i), 1);
    fence_mbar_init();
    ctl.abort = 0;
  }
  if (threadIdx.x < D / 2) ctl.om[threadIdx.x] = a.inv_freq[threadIdx.x];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;
  grid_dependency_wait();          // q', k' (summary kernel) and the reverse index come from earlier kernels
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }

  constexpr uint32_t idS = idesc_bf16_f32(BS, BS, 0, 0);
  constexpr uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);
  const float sl2 = a.scale * 1.4426950408889634f;
  const long long ntiles = static_cast<long long>(a.B) * a.Hq * a.nb;
  const int g = a.Hq / a.Hkv;
  uint32_t phQ = 0, phS = 0, phMM = 0;
  long long ld_issue = 0, ld_use = 0;             // (K, V) loads: slot = n % NKV, parity (n / NKV) & 1
  bool mm_pending = false, ok = true, q_pending = false;
  int mm_step = 0;

  const uint64_t t_start = globaltimer();
  // Wait for a barrier phase in every thread; false (everywhere) if any gave
  // up or the CTA's time budget ran out; the site is recorded.
  auto wait_all = [&](int bar, uint32_t parity, int site) -> bool {
    const bool w = mbar_wait(BAR(bar), parity, kBwWaitNs);
    const bool in_time = globaltimer() - t_start <= kBwBudgetNs;
    if (!(w && in_time)) record_site(a.status, 100 + site + (w ? 50 : 0));
    return __syncthreads_and(w && in_time) != 0;
  };

  for (long long tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
    const int j = static_cast<int>(tile % a.nb), hq = static_cast<int>((tile / a.nb) % a.Hq);
    const int b = static_cast<int>(tile / (static_cast<long long>(a.nb) * a.Hq));
    const int h = hq / g;
    __syncthreads();                              // the previous tile's ids are no longer read
    if (R.warp == 0) {
      const int32_t* row = a.sel + tile * a.nsel;
      const int e0 = R.lane < a.nsel ? row[R.lane] : -1, e1 = R.lane + 32 < a.nsel ? row[R.lane + 32] : -1;
      const bool v0 = e0 >= 0 && e0 <= j, v1 = e1 >= 0 && e1 <= j;
      if (e0 > j || e1 > j) atomicExch(a.status, kDevBadSelection);
      const unsigned m0 = __ballot_sync(0xffffffffu, v0), m1 = __ballot_sync(0xffffffffu, v1);
      const unsigned lt = (1u << R.lane) - 1u;
      if (v0) ctl.ids[__popc(m0 & lt)] = static_cast<int16_t>(e0);
      if (v1) ctl.ids[__popc(m0) + __popc(m1 & lt)] = static_cast<int16_t>(e1);
      if (R.lane == 0) ctl.nblk = __popc(m0) + __popc(m1);
    }
    __syncthreads();
    const int nblk = ctl.nblk;
    const long long tok0 = static_cast<long long>(b) * a.S + static_cast<long long>(j) * BS;
    const long long si0 = (static_cast<long long>(b) * a.Hq + hq) * a.S + static_cast<long long>(j) * BS;
    if (nblk == 0) {                              // nothing selected: zero gradient, no row statistics
      for (int e = threadIdx.x; e < BS * D; e += kBwThreads)
        a.dq[((tok0 + e / D) * a.Hq + hq) * D + e % D] = 0.f;
      for (int t = threadIdx.x; t < BS; t += kBwThreads) {
        a.lse[si0 + t] = INFINITY;
        a.delta[si0 + t] = 0.f;
      }
      continue;
    }
    // Pass 1 then pass 2 over the same blocks; with the forward's output and
    // row normalisers given, pass 2 alone.
    const bool given = a.lse_in != nullptr;
    const int p2 = given ? 0 : nblk;
    const int nsteps = p2 + nblk;
    auto issue_kv = [&](int n) {                  // K, V of step n into slot ld_issue % NKV
      if (threadIdx.x == 0) {
        const int slot = static_cast<int>(ld_issue % C::NKV);
        const uint32_t bar = BAR(bKV0 + slot), dst = sKV + slot * 2 * C::kTile;
        const int blk = ctl.ids[n % nblk];
        mbar_expect_tx(bar, 2 * C::kTile);
#pragma unroll
        for (int gg = 0; gg < D / 64; ++gg) {
          tma_load_3d(dst + gg * C::kRegion, &tmK, bar, gg * 64, h, static_cast<int>(b * a.S + blk * BS));
          tma_load_3d(dst + C::kTile + gg * C::kRegion, &tmV, bar, gg * 64, h, static_cast<int>(b * a.S + blk * BS));
        }
      }
      ++ld_issue;
    };
    // The MMA of step mm_step (PV or dQ) has completed: its slot is free for
    // step mm_step + NKV.
    auto finish_mm = [&]() -> bool {
      if (!mm_pending) return true;
      if (!wait_all(bMM, phMM, kSiteMM)) return false;
      phMM ^= 1;
      mm_pending = false;
      if (mm_step + C::NKV < nsteps) issue_kv(mm_step + C::NKV);
      return true;
    };
    if (threadIdx.x == 0) {
      mbar_expect_tx(BAR(bQ), 2 * C::kTile);
#pragma unroll
      for (int gg = 0; gg < D / 64; ++gg) {
        tma_load_3d(sQ + gg * C::kRegion, &tmQ, BAR(bQ), gg * 64, hq, static_cast<int>(tok0));
        tma_load_3d(sO + gg * C::kRegion, &tmO, BAR(bQ), gg * 64, hq, static_cast<int>(tok0));
      }
    }
    q_pending = true;
    for (int n = 0; n < C::NKV && n < nsteps; ++n) issue_kv(n);
    if (!wait_all(bQ, phQ, kSiteQ)) { ok = false; break; }
    phQ ^= 1;
    q_pending = false;
    float m2 = -INFINITY, l = 0.f, lse2 = 0.f, delta = 0.f;
    if (given) {
      // Delta = <dO, out> of the saved (normalised) output; lse in log2 units.
      const __nv_bfloat16* dorow = static_cast<const __nv_bfloat16*>(a.dout) + ((tok0 + R.r) * a.Hq + hq) * D;
      const __nv_bfloat16* orow = static_cast<const __nv_bfloat16*>(a.out_in) + ((tok0 + R.r) * a.Hq + hq) * D;
      float dsum = 0.f;
#pragma unroll
      for (int pp = 0; pp < C::NP; ++pp)
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int c0 = (hf ? D / 2 : 0) + R.col_lo(pp);
          float o[C::W];
#pragma unroll
          for (int q = 0; q < C::W / 8; ++q) Elem<__nv_bfloat16>::load(orow + c0 + 8 * q, o + 8 * q);
          dsum += dot_bf16<C::W>(o, dorow + c0);
        }
      delta = R.row_sum(dsum);
      const float ln = a.lse_in[si0 + R.r];
      lse2 = ln > -INFINITY ? ln * 1.4426950408889634f : INFINITY;
      if (R.tsub == 0) {
        a.lse[si0 + R.r] = lse2;
        a.delta[si0 + R.r] = delta;
      }
    }
    for (int n = 0; n < nsteps && ok; ++n) {
      const bool pass2 = n >= p2;
      const int blk = ctl.ids[n % nblk];
      const int slot = static_cast<int>(ld_use % C::NKV);
      if (!wait_all(bKV0 + slot, static_cast<uint32_t>((ld_use / C::NKV) & 1), kSiteKV)) { ok = false; break; }
      ++ld_use;
      const uint32_t sK = sKV + slot * 2 * C::kTile, sV = sK + C::kTile;
      if (threadIdx.x == 0) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) mma_bf16(tmem + C::qColS, kmaj<BS>(sQ, kk), kmaj<BS>(sK, kk), idS, kk > 0);
        if (pass2) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) mma_bf16(tmem + C::qColP, kmaj<BS>(sO, kk), kmaj<BS>(sV, kk), idS, kk > 0);
        }
        mma_commit(BAR(bS));
      }
      if (!wait_all(bS, phS, kSiteS)) { ok = false; break; }
      phS ^= 1;
      if (!finish_mm()) { ok = false; break; }     // O (or dQ) and the P buffer are free
      tc_fence_after();
      const bool diag = blk == j;
      if (!pass2) {
        // Row maximum of this block, then rescale O and the sum if it grew.
        float mx = -INFINITY;
        float sv[C::NC][32];
#pragma unroll
        for (int c = 0; c < C::NC; ++c) {
          const int k0 = R.ld_scores(tmem + C::qColS, c, sv[c]);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            sv[c][e] = (diag && k0 + e > R.r) ? -INFINITY : sv[c][e] * sl2;
            mx = fmaxf(mx, sv[c][e]);
          }
        }
        mx = R.row_max(mx);
        const bool grow = mx > m2;
        const float alpha = (grow && n > 0) ? ex2(m2 - mx) : 1.f;   // 1 for rows whose maximum stays
        if (grow) {
          l *= alpha;
          m2 = mx;
        }
        // tcgen05.ld / tcgen05.st are warp-collective (.sync.aligned): the
        // whole warp rescales its rows' O when any of them grew, the others
        // by 1, so no lane skips an instruction another lane executes.
        if (n > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int pp = 0; pp < C::NP; ++pp)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              float o[C::W];
              R.ld_d(tmem + C::qColO, pp, hf, o);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < C::W; ++e) o[e] *= alpha;
              R.st_d(tmem + C::qColO, pp, hf, o);
            }
          tmem_st_wait();
        }
        const float mref = m2 == -INFINITY ? 0.f : m2;   // a row with no visible key yet gets P = 0
#pragma unroll
        for (int c = 0; c < C::NC; ++c) {
          const int k0 = C::kHR ? 32 * R.tsub : 32 * c;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float p[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              p[e] = ex2(sv[c][8 * q + e] - mref);
              l += p[e];
            }
            st_bf16x8<BS>(pP, R.r, k0 + 8 * q, p);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < C::NC; ++c) {
          float sv[32], dp[32];
          const int k0 = R.ld_scores(tmem + C::qColS, c, sv);
          R.ld_scores(tmem + C::qColP, c, dp);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float ds[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int k = k0 + 8 * q + e;
              const float p = (diag && k > R.r) ? 0.f : ex2(sv[8 * q + e] * sl2 - lse2);
              ds[e] = p * (dp[8 * q + e] - delta);
            }
            st_bf16x8<BS>(pP, R.r, k0 + 8 * q, ds);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();
      if (threadIdx.x == 0) {
        tc_fence_after();
        // pass 1: O += P V (V MN-major); pass 2: dQ += dS K (K MN-major)
        const uint32_t sB = pass2 ? sK : sV;
        const bool first = n == (pass2 ? p2 : 0);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          mma_bf16(tmem + C::qColO, kmaj<BS>(sP, kk), mnmaj<BS>(sB, kk), idPV, (!first || kk > 0) ? 1u : 0u);
        mma_commit(BAR(bMM));
      }
      mm_pending = true;
      mm_step = n;
      if (!given && n == nblk - 1) {
        // End of pass 1: lse and Delta = <dO, O> / sum of each row.
        if (!finish_mm()) { ok = false; break; }
        tc_fence_after();
        const float lt = R.row_sum(l);
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const __nv_bfloat16* dorow = static_cast<const __nv_bfloat16*>(a.dout) + ((tok0 + R.r) * a.Hq + hq) * D;
        float dsum = 0.f;
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            float o[C::W];
            R.ld_d(tmem + C::qColO, pp, hf, o);
            tmem_ld_wait();
            dsum += dot_bf16<C::W>(o, dorow + (hf ? D / 2 : 0) + R.col_lo(pp));
          }
        delta = R.row_sum(dsum) * inv;
        lse2 = lt > 0.f ? m2 + __log2f(lt) : INFINITY;
        if (R.tsub == 0) {
          a.lse[si0 + R.r] = lse2;
          a.delta[si0 + R.r] = delta;
        }
      } else if (n == nsteps - 1) {
        // End of pass 2: dq = R(t)^T (scale dQ).
        if (!finish_mm()) { ok = false; break; }
        tc_fence_after();
        float* dqrow = a.dq + ((tok0 + R.r) * a.Hq + hq) * D;
        const int t = j * BS + R.r;
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp) {
          float lo[C::W], hi[C::W];
          R.ld_d(tmem + C::qColO, pp, 0, lo);
          R.ld_d(tmem + C::qColO, pp, 1, hi);
          tmem_ld_wait();
          rotate_store<C::W, D>(lo, hi, R.col_lo(pp), t, a.scale, ctl.om, dqrow);
        }
      }
    }
    tc_fence_before();
  }

  if (!ok) {
    if (threadIdx.x == 0) {
      atomicExch(a.status, kDevWaitTimeout);
      mma_commit(BAR(bFin));                      // arrives once every MMA issued so far is done
      mbar_wait(BAR(bFin), 0, kBwWaitNs);
      for (long long n = ld_use; n < ld_issue; ++n)
        mbar_wait(BAR(bKV0 + static_cast<int>(n % C::NKV)), static_cast<uint32_t>((n / C::NKV) & 1), kBwWaitNs);
      if (q_pending) mbar_wait(BAR(bQ), phQ, kBwWaitNs);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (R.warp == 0) {
    __syncwarp();
    tmem_dealloc(tmem, C::qCols);
  }
}

// ------------------------------------------- dk/dv kernel, warp-specialised
// Roles: warps 0-7 compute P^T and dS^T (warp w reads TMEM subpartition
// w % 4 and half w / 4 of each entry's columns; warps 0-3 also run the
// epilogue), warp 8 loads by TMA, warp 9 issues the MMAs (and owns the
// tensor memory).
// S^T and dP^T of the next entry are computed while the four warps work on
// the current one (two TMEM buffers at bs = 64); the next key tile's K and V
// load into a second buffer during the current tile (not at bs = D = 128),
// and at bs = 64 the epilogue hands the accumulators back as soon as it has
// read them; every hand-off is an
// mbarrier, every wait bounded (2 s, and given up as soon as another role has
// given up).
constexpr int kWsThreads = 320;                  // 8 elementwise warps, a TMA warp, an MMA warp
constexpr int kWsEw = 8;                         // elementwise warps: two per TMEM subpartition

template <int BS, int D>
struct WsCfg {
  using C = BwCfg<BS, D>;
  static constexpr int NS = (BS == 64) ? 2 : 1;                       // S^T / dP^T / P^T / dS^T buffers
  static constexpr int NE = (BS == 64) ? (D == 64 ? 8 : 3) : (D == 64 ? 2 : 1);   // entry slots
  // (K, V) tile buffers: two, so that the next key tile's K and V (and, behind
  // them, its entries) load while the current tile is processed; one at
  // bs = D = 128, where a second does not fit.
  static constexpr int NKV = (BS == 128 && D == 128) ? 1 : 2;
  static constexpr int kSlot = C::kSlot;
  static constexpr int kHdr = 2 * C::kTile + 2 * BS * 4;               // the entry's query block (int)
  static_assert(kHdr + 4 <= kSlot, "entry slot header");
  static constexpr int oKV = 0, oE = NKV * 2 * C::kTile;
  static constexpr int oPT = oE + NE * kSlot;                          // NS x P^T
  static constexpr int oDS = oPT + NS * C::kPTile;                     // NS x dS^T
  static constexpr int oCtl = oDS + NS * C::kPTile;
  static constexpr int kSmem = oCtl + 1024;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static constexpr int colS = 0, colP = NS * BS, colV = 2 * NS * BS, colK = 2 * NS * BS + D;
  static constexpr int kCols = pow2_cols(2 * NS * BS + 2 * D);
  static_assert(2 * NS * BS + 2 * D <= 512, "tensor memory");
  // barriers
  static constexpr int bKvF = 0, bKvE = 2, bAF = 4, bAE = 5, bFin = 6;   // bKvF, bKvE: NKV each
  static constexpr int bEF = 7, bEE = bEF + NE;
  static constexpr int bSF = bEE + NE, bSE = bSF + NS, bPF = bSE + NS, bPE = bPF + NS;
  static constexpr int kBars = bPE + NS;
  static_assert(kBars <= 32, "barrier space");
};

struct WsCtl {
  uint64_t bar[32];
  float om[64];
  uint32_t tmem;
  int abort;
};

template <int BS, int D>
__global__ void __launch_bounds__(kWsThreads, 1)
bwd_dkdv_ws_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const BwdArgs a) {
  using C = BwCfg<BS, D>;
  using W = WsCfg<BS, D>;
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(a.status, kDevMisaligned);
    return;
  }
  WsCtl& ctl = *reinterpret_cast<WsCtl*>(smem + W::oCtl);
  const uint32_t base = smem_u32(smem);
  const uint32_t sKV = base + W::oKV, sE = base + W::oE;
  auto BAR = [&](int i) { return smem_u32(&ctl.bar[i]); };
  volatile int* abort_flag = &ctl.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == kWsEw + 1) {
    tmem_alloc(smem_u32(&ctl.tmem), W::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < W::kBars; ++i) {
      int count = 1;
      if (i == W::bAE) count = 4;                                        // the epilogue warps
      if ((i >= W::bSE && i < W::bSE + W::NS) || (i >= W::bPF && i < W::bPF + W::NS)) count = kWsEw;
      mbar_init(BAR(i), count);
    }
    fence_mbar_init();
    ctl.abort = 0;
  }
  if (threadIdx.x < D / 2) ctl.om[threadIdx.x] = a.inv_freq[threadIdx.x];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem;
  grid_dependency_wait();          // lse, Delta (dq kernel) and the reverse index come from earlier kernels

  const long long nkt = static_cast<long long>(a.B) * a.Hkv * a.nb;
  const int g = a.Hq / a.Hkv;
  const long long E = static_cast<long long>(g) * a.nb * a.nsel;
  // Entries of key tile kt (0 for a reverse-index range that is out of bounds,
  // which a reverse index of this call never gives; recorded).
  auto entries = [&](long long kt, int* e0_out) -> int {
    const int i = static_cast<int>(kt % a.nb);
    const long long bh = kt / a.nb;
    const int32_t* roff = a.rev_off + bh * (a.nb + 1);
    const int e0 = roff[i], ne = roff[i + 1] - e0;
    *e0_out = e0;
    if (e0 < 0 || ne < 0 || e0 + static_cast<long long>(ne) > E) {
      if (threadIdx.x == 0 || threadIdx.x == 32 * kWsEw) {
        atomicExch(a.status, kDevBadSelection);
        record_site(a.status, 200 + kSiteRevRange);
      }
      return 0;
    }
    return ne;
  };
  auto code_of = [&](const int32_t* rev, int e) -> int {
    int code = rev[e];
    if (code < 0 || code >= g * a.nb) {
      atomicExch(a.status, kDevBadSelection);
      record_site(a.status, 200 + kSiteRevCode);
      code = 0;
    }
    return code;
  };
  auto fail = [&](int site) {
    atomicExch(a.status, kDevWaitTimeout);
    record_site(a.status, 200 + site);
    *abort_flag = 1;
  };
  auto waitb = [&](int bar, uint32_t parity) -> bool {
    if (mbar_try_wait(BAR(bar), parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
      for (int k = 0; k < 32; ++k)
        if (mbar_try_wait(BAR(bar), parity)) return true;
      if (*abort_flag) return false;
      if (globaltimer() - t0 > kBwWaitNs) return false;
    }
  };

  if (warp == kWsEw) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      prefetch_tmap(&tmO);
      long long xg = 0, tc_ = 0, kv_issued = 0;   // entries, key tiles, key tiles whose K, V were issued
      bool ok = true;
      for (long long kt = blockIdx.x; kt < nkt && ok; kt += gridDim.x) {
        int e0;
        const int ne = entries(kt, &e0);
        if (ne == 0) continue;
        const int i = static_cast<int>(kt % a.nb);
        const long long bh = kt / a.nb;
        const int h = static_cast<int>(bh % a.Hkv), b = static_cast<int>(bh / a.Hkv);
        const int32_t* rev = a.rev + bh * E;
        const int kv = static_cast<int>(tc_ % W::NKV);
        if (tc_ >= W::NKV &&
            !waitb(W::bKvE + kv, static_cast<uint32_t>(((tc_ / W::NKV) - 1) & 1))) { fail(kSiteKV); ok = false; break; }
        const int row0 = static_cast<int>(static_cast<long long>(b) * a.S + static_cast<long long>(i) * BS);
        const uint32_t sKb = sKV + kv * 2 * C::kTile, kvbar = BAR(W::bKvF + kv);
        mbar_expect_tx(kvbar, 2 * C::kTile);
        kv_issued = tc_ + 1;
#pragma unroll
        for (int gg = 0; gg < D / 64; ++gg) {
          tma_load_3d(sKb + gg * C::kRegion, &tmK, kvbar, gg * 64, h, row0);
          tma_load_3d(sKb + C::kTile + gg * C::kRegion, &tmV, kvbar, gg * 64, h, row0);
        }
        for (int x = 0; x < ne; ++x, ++xg) {
          const int slot = static_cast<int>(xg % W::NE);
          if (xg >= W::NE && !waitb(W::bEE + slot, static_cast<uint32_t>(((xg / W::NE) - 1) & 1))) {
            fail(kSiteEntry);
            ok = false;
            break;
          }
          const int code = code_of(rev, e0 + x);
          const int hl = code / a.nb, jq = code - hl * a.nb, hq = h * g + hl;
          const uint32_t bar = BAR(W::bEF + slot), dst = sE + slot * W::kSlot;
          const int q0 = static_cast<int>(static_cast<long long>(b) * a.S + static_cast<long long>(jq) * BS);
          const long long si0 = (static_cast<long long>(b) * a.Hq + hq) * a.S + static_cast<long long>(jq) * BS;
          // The entry's query block, for the elementwise warps: published by
          // the full barrier's arrive below.
          *reinterpret_cast<volatile int*>(smem + W::oE + slot * W::kSlot + W::kHdr) = jq;
          mbar_expect_tx(bar, 2 * C::kTile + 2 * BS * 4);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg) {
            tma_load_3d(dst + gg * C::kRegion, &tmQ, bar, gg * 64, hq, q0);
            tma_load_3d(dst + C::kTile + gg * C::kRegion, &tmO, bar, gg * 64, hq, q0);
          }
          bulk_load(dst + 2 * C::kTile, a.lse + si0, BS * 4, bar);
          bulk_load(dst + 2 * C::kTile + BS * 4, a.delta + si0, BS * 4, bar);
        }
        ++tc_;
      }
      if (!ok) {
        // Wait (bounded) for the copies this thread issued and nobody consumed.
        for (long long n = kv_issued - W::NKV > 0 ? kv_issued - W::NKV : 0; n < kv_issued; ++n)
          mbar_wait(BAR(W::bKvF + static_cast<int>(n % W::NKV)), static_cast<uint32_t>((n / W::NKV) & 1), kBwWaitNs);
        for (long long n = xg - W::NE > 0 ? xg - W::NE : 0; n < xg; ++n)
          mbar_wait(BAR(W::bEF + static_cast<int>(n % W::NE)), static_cast<uint32_t>((n / W::NE) & 1), kBwWaitNs);
      }
    }
  } else if (warp == kWsEw + 1) {
    // ------------------------------------------------------------- MMAs
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BS, BS, 0, 0);
      constexpr uint32_t idG = idesc_bf16_f32(BS, D, 0, 1);
      long long xg = 0, tc_ = 0;
      bool ok = true;
      // dV += P^T dO, dK += dS^T Q for entry yg (x-th of its tile).
      auto acc = [&](long long yg, int y) -> bool {
        const int pb = static_cast<int>(yg % W::NS), slot = static_cast<int>(yg % W::NE);
        if (!waitb(W::bPF + pb, static_cast<uint32_t>((yg / W::NS) & 1))) { fail(kSiteMM); return false; }
        if (y == 0 && tc_ > 0 && !waitb(W::bAE, static_cast<uint32_t>((tc_ - 1) & 1))) { fail(kSiteMM); return false; }
        tc_fence_after();
        const uint32_t sQe = sE + slot * W::kSlot, sOe = sQe + C::kTile;
        const uint32_t sPT = base + W::oPT + pb * C::kPTile, sDS = base + W::oDS + pb * C::kPTile;
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          mma_bf16(tmem + W::colV, kmaj<BS>(sPT, kk), mnmaj<BS>(sOe, kk), idG, (y > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          mma_bf16(tmem + W::colK, kmaj<BS>(sDS, kk), mnmaj<BS>(sQe, kk), idG, (y > 0 || kk > 0) ? 1u : 0u);
        mma_commit(BAR(W::bPE + pb));
        mma_commit(BAR(W::bEE + slot));
        return true;
      };
      // The next tile's reverse-list offsets are read a tile ahead, so that
      // their latency does not sit between two tiles' products.
      auto offsets = [&](long long kt, int* lo, int* hi) {
        if (kt >= nkt) { *lo = *hi = 0; return; }
        const int32_t* roff = a.rev_off + (kt / a.nb) * (a.nb + 1) + kt % a.nb;
        *lo = roff[0];
        *hi = roff[1];
      };
      int nlo, nhi;
      offsets(blockIdx.x, &nlo, &nhi);
      for (long long kt = blockIdx.x; kt < nkt && ok; kt += gridDim.x) {
        const int e0 = nlo, e1 = nhi;
        offsets(kt + gridDim.x, &nlo, &nhi);
        // The same range checks as entries(), which the other roles run.
        const int ne = (e0 < 0 || e1 < e0 || e1 > E) ? 0 : e1 - e0;
        if (ne == 0) continue;
        const int kv = static_cast<int>(tc_ % W::NKV);
        if (!waitb(W::bKvF + kv, static_cast<uint32_t>((tc_ / W::NKV) & 1))) { fail(kSiteKV); ok = false; break; }
        const uint32_t sK = sKV + kv * 2 * C::kTile, sV = sK + C::kTile;
        for (int x = 0; x < ne; ++x, ++xg) {
          const int slot = static_cast<int>(xg % W::NE), sb = static_cast<int>(xg % W::NS);
          // With a single entry slot, entry x loads only once entry x-1's
          // products have read the slot: issue those first.
          if (W::NE == 1 && x > 0 && !acc(xg - 1, x - 1)) { ok = false; break; }
          if (!waitb(W::bEF + slot, static_cast<uint32_t>((xg / W::NE) & 1))) { fail(kSiteEntry); ok = false; break; }
          if (xg >= W::NS && !waitb(W::bSE + sb, static_cast<uint32_t>(((xg / W::NS) - 1) & 1))) {
            fail(kSiteS);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sQe = sE + slot * W::kSlot, sOe = sQe + C::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16(tmem + W::colS + sb * BS, kmaj<BS>(sK, kk), kmaj<BS>(sQe, kk), idS, kk > 0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16(tmem + W::colP + sb * BS, kmaj<BS>(sV, kk), kmaj<BS>(sOe, kk), idS, kk > 0);
          mma_commit(BAR(W::bSF + sb));
          if (W::NE > 1 && x > 0 && !acc(xg - 1, x - 1)) { ok = false; break; }
        }
        if (!ok) break;
        if (!acc(xg - 1, ne - 1)) { ok = false; break; }
        mma_commit(BAR(W::bAF));
        mma_commit(BAR(W::bKvE + static_cast<int>(tc_ % W::NKV)));
        ++tc_;
      }
      // Everything this thread issued has completed once bFin fires.
      mma_commit(BAR(W::bFin));
      mbar_wait(BAR(W::bFin), 0, kBwWaitNs);
    }
  } else {
    // ---------------------------------------------- P^T, dS^T, epilogue
    const Rows<BS, D> R;                             // TMEM subpartition warp % 4
    const int ch = warp >> 2;                        // which half of an entry's columns
    const float sl2 = a.scale * 1.4426950408889634f;
    auto wwait = [&](int bar, uint32_t parity) { return __all_sync(0xffffffffu, waitb(bar, parity)) != 0; };
    long long xg = 0, tc_ = 0;
    bool ok = true;
    for (long long kt = blockIdx.x; kt < nkt && ok; kt += gridDim.x) {
      int e0;
      const int ne = entries(kt, &e0);
      const int i = static_cast<int>(kt % a.nb);
      const long long bh = kt / a.nb;
      const int h = static_cast<int>(bh % a.Hkv), b = static_cast<int>(bh / a.Hkv);
      const long long tok0 = static_cast<long long>(b) * a.S + static_cast<long long>(i) * BS;
      if (ne == 0) {                                // no query selected this block
        for (int e = threadIdx.x; e < BS * D; e += 32 * kWsEw) {
          const long long o = ((tok0 + e / D) * a.Hkv + h) * D + e % D;
          a.dk[o] = 0.f;
          a.dv[o] = 0.f;
        }
        continue;
      }
      for (int x = 0; x < ne; ++x, ++xg) {
        const int sb = static_cast<int>(xg % W::NS), slot = static_cast<int>(xg % W::NE);
        if (!wwait(W::bSF + sb, static_cast<uint32_t>((xg / W::NS) & 1))) { ok = false; break; }
        if (!wwait(W::bEF + slot, static_cast<uint32_t>((xg / W::NE) & 1))) { ok = false; break; }   // lse, Delta landed
        tc_fence_after();
        const int jq = *reinterpret_cast<volatile const int*>(smem + W::oE + slot * W::kSlot + W::kHdr);
        const bool diag = jq == i;
        const float* lse_s = reinterpret_cast<const float*>(smem + W::oE + slot * W::kSlot + 2 * C::kTile);
        const float* del_s = lse_s + BS;
        uint8_t* pPT = smem + W::oPT + sb * C::kPTile;
        uint8_t* pDS = smem + W::oDS + sb * C::kPTile;
        // P^T, dS^T of NW columns from t0 into the shared-memory operands.
        auto cols_out = [&](const float* sv, const float* dp, int t0, auto nw) {
          constexpr int NW = decltype(nw)::value;
#pragma unroll
          for (int q = 0; q < NW / 8; ++q) {
            float p[8], ds[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int t = t0 + 8 * q + e;
              p[e] = (diag && t < R.r) ? 0.f : ex2(sv[8 * q + e] * sl2 - lse_s[t]);
              ds[e] = p[e] * (dp[8 * q + e] - del_s[t]);
            }
            st_bf16x8<BS>(pPT, R.r, t0 + 8 * q, p);
            st_bf16x8<BS>(pDS, R.r, t0 + 8 * q, ds);
          }
        };
        if constexpr (C::NC == 1) {
          // bs = 64: 16 columns a thread (32 ch + 16 tsub ..); free the S^T,
          // dP^T buffer before waiting for the P^T, dS^T buffer, so the next
          // entry's products can start.
          float sv[16], dp[16];
          tmem_ld16x2_16(tmem + W::colS + sb * BS + 32 * ch + R.lane_base, sv);
          tmem_ld16x2_16(tmem + W::colP + sb * BS + 32 * ch + R.lane_base, dp);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(W::bSE + sb));          // S^T, dP^T buffer free
          if (xg >= W::NS && !wwait(W::bPE + sb, static_cast<uint32_t>(((xg / W::NS) - 1) & 1))) { ok = false; break; }
          cols_out(sv, dp, 32 * ch + 16 * R.tsub, std::integral_constant<int, 16>{});
        } else {
          // bs = 128 (one buffer): chunks 2 ch and 2 ch + 1 of 32 columns.
          if (xg >= W::NS && !wwait(W::bPE + sb, static_cast<uint32_t>(((xg / W::NS) - 1) & 1))) { ok = false; break; }
#pragma unroll 1
          for (int c = 2 * ch; c < 2 * ch + 2; ++c) {
            float sv[32], dp[32];
            const int t0 = R.ld_scores(tmem + W::colS + sb * BS, c, sv);
            R.ld_scores(tmem + W::colP + sb * BS, c, dp);
            tmem_ld_wait();
            cols_out(sv, dp, t0, std::integral_constant<int, 32>{});
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(W::bSE + sb));          // S^T, dP^T buffer free
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(W::bPF + sb));
      }
      if (!ok) break;
      ++tc_;
      if (ch != 0) continue;                           // the epilogue: warps 0-3
      // dv = dV; dk = R(s)^T (scale dK).
      if (!wwait(W::bAF, static_cast<uint32_t>((tc_ - 1) & 1))) { ok = false; break; }
      tc_fence_after();
      const long long krow = (tok0 + R.r) * a.Hkv + h;
      const int s = i * BS + R.r;
      if constexpr (C::NP == 1) {
        // One part per thread: read both accumulators, hand them back to the
        // MMA lane at once (the next tile's products may start), then store.
        float vlo[C::W], vhi[C::W], klo[C::W], khi[C::W];
        R.ld_d(tmem + W::colV, 0, 0, vlo);
        R.ld_d(tmem + W::colV, 0, 1, vhi);
        R.ld_d(tmem + W::colK, 0, 0, klo);
        R.ld_d(tmem + W::colK, 0, 1, khi);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(W::bAE));
        store_f32<C::W>(a.dv + krow * D + R.col_lo(0), vlo);
        store_f32<C::W>(a.dv + krow * D + D / 2 + R.col_lo(0), vhi);
        rotate_store<C::W, D>(klo, khi, R.col_lo(0), s, a.scale, ctl.om, a.dk + krow * D);
      } else {
#pragma unroll
        for (int pp = 0; pp < C::NP; ++pp) {
          float lo[C::W], hi[C::W];
          R.ld_d(tmem + W::colV, pp, 0, lo);
          R.ld_d(tmem + W::colV, pp, 1, hi);
          tmem_ld_wait();
          store_f32<C::W>(a.dv + krow * D + R.col_lo(pp), lo);
          store_f32<C::W>(a.dv + krow * D + D / 2 + R.col_lo(pp), hi);
          R.ld_d(tmem + W::colK, pp, 0, lo);
          R.ld_d(tmem + W::colK, pp, 1, hi);
          tmem_ld_wait();
          rotate_store<C::W, D>(lo, hi, R.col_lo(pp), s, a.scale, ctl.om, a.dk + krow * D);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(W::bAE));
      }
    }
    if (!ok && lane == 0) fail(kSiteS);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWsEw + 1) {
    __syncwarp();
    tmem_dealloc(tmem, W::kCols);
  }
}

namespace {

template <typename K>
cudaError_t launch_persistent(K kernel, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                              const CUtensorMap& mo, const BwdArgs& a, long long ntiles, int smem, int cols,
                              int threads, cudaStream_t st) {
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(kernel), smem);
  if (e != cudaSuccess) return e;
  // All of the unified L1 / shared storage as shared memory (these kernels
  // read their operands through TMA, not L1).
  e = cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int sms = cached_sm_count();
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(kernel), threads, smem);
  if (sms <= 0) return cudaErrorUnknown;
  // Residency from the kernel's own registers and shared memory (the larger
  // of this and the occupancy query; a CTA that does not fit waits for one
  // to finish, so an overestimate costs nothing).
  {
    int dev = 0, regs_sm = 0, smem_sm = 0, reserved = 0;
    cudaFuncAttributes fa{};
    if (cudaGetDevice(&dev) == cudaSuccess && cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(kernel)) == cudaSuccess &&
        cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev) == cudaSuccess) {
      const int warps = (threads + 31) / 32;
      const int regs_warp = (fa.numRegs * 32 + 255) / 256 * 256;
      const int by_regs = regs_sm / (regs_warp * warps);
      const int by_smem = smem_sm / (smem + static_cast<int>(fa.sharedSizeBytes) + reserved);
      int est = by_regs < by_smem ? by_regs : by_smem;
      if (est > per_sm) per_sm = est;
    }
  }
  per_sm = per_sm < 512 / cols ? per_sm : 512 / cols;    // tensor memory: 512 columns per SM
  if (per_sm < 1) per_sm = 1;
  const long long want = static_cast<long long>(sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(ntiles < want ? ntiles : want);
  if (grid == 0) return cudaSuccess;
  return launch_pdl(kernel, dim3(grid), dim3(threads), static_cast<size_t>(smem), st, mq, mk, mv, mo, a);
}

template <int BS, int D>
cudaError_t launch_tc_bwd(const BwdArgs& a, cudaStream_t st) {
  using C = BwCfg<BS, D>;
  CUtensorMap mq, mk, mv, mo;
  const long long rows = static_cast<long long>(a.B) * a.S;
  if (!make_tile_map(&mq, a.qrot, rows, a.Hq, D, BS) || !make_tile_map(&mk, a.krot, rows, a.Hkv, D, BS) ||
      !make_tile_map(&mv, a.v, rows, a.Hkv, D, BS) || !make_tile_map(&mo, a.dout, rows, a.Hq, D, BS))
    return cudaErrorInvalidValue;
  cudaError_t e = launch_persistent(bwd_dq_tc_kernel<BS, D>, mq, mk, mv, mo, a,
                                    static_cast<long long>(a.B) * a.Hq * a.nb, C::qSmem, C::qCols, kBwThreads, st);
  if (e != cudaSuccess) return e;
  using W = WsCfg<BS, D>;
  return launch_persistent(bwd_dkdv_ws_kernel<BS, D>, mq, mk, mv, mo, a,
                           static_cast<long long>(a.B) * a.Hkv * a.nb, W::kSmem, W::kCols, kWsThreads, st);
}

}  // namespace

cudaError_t launch_backward_tc(const BwdArgs& a, cudaStream_t st) {
  cudaError_t e = launch_bwd_rev(a, st);
  if (e != cudaSuccess) return e;
  if (a.bs == 64 && a.D == 64) e = launch_tc_bwd<64, 64>(a, st);
  else if (a.bs == 64 && a.D == 128) e = launch_tc_bwd<64, 128>(a, st);
  else if (a.bs == 128 && a.D == 64) e = launch_tc_bwd<128, 64>(a, st);
  else if (a.bs == 128 && a.D == 128) e = launch_tc_bwd<128, 128>(a, st);
  else return cudaErrorInvalidValue;
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
