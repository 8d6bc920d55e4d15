// K5 (tensor cores): selected-set causal attention, bf16, on tcgen05 + TMEM.
//
// For token t of query block j and query head hq: softmax over every token s
// of the blocks listed in sel[b,hq,j] with s <= t of scale * <q'_t, k'_s>,
// applied to v_s ("Monodratic: a reproducible sparse attention mixer",
// section Mixer: exact causal softmax over the selected set, with the
// selected values themselves).
//
// Persistent, warp-specialised kernel.  A CTA walks the (b, hq, j) tiles
// blockIdx.x, blockIdx.x + gridDim.x, ...  (consecutive CTAs take
// consecutive query blocks of one head, so that head's K/V stays in L2).
//   warp 0        TMA producers: lane 0 loads the Q tile of each query block
//                 into a Q ring and the K tile of every selected block into a
//                 K ring, lane 1 the V tiles into a V ring (128-byte swizzle,
//                 mbarrier expect-tx).  A K stage is refilled once the S MMA
//                 that read it completed, a V stage once its PV completed.
//   warp 1        MMA issuer (one lane): S = Q K^T (M = bs, N = bs, K = D)
//                 into one of two TMEM S buffers, and O += P V (M = bs,
//                 N = D, K = bs keys; V read MN-major from its TMA tile)
//                 into the TMEM O accumulator.  S of block n+2 is issued as
//                 soon as the softmax has consumed S of block n, so the
//                 tensor core works on the next scores and the previous PV
//                 while the softmax runs.
//   warps 2..5    softmax: one query row per thread (tcgen05.ld), causal
//                 mask inside the query's own block, running maximum and
//                 sum in float32 (log2 units), P = exp(S - max) as bf16 into
//                 one of two shared-memory P buffers in the K-major swizzled
//                 layout the PV MMA reads; O is rescaled in TMEM only when the
//                 running maximum grows by more than 2^8 (exact, since the
//                 final division uses the same maximum); epilogue O / sum ->
//                 bf16 -> global.
// TMEM accumulators with M = 64 keep row r in lane (r % 16) + 32 (r / 16); with
// M = 128 in lane r.  Warp w may only touch lanes 32 (w % 4) .. + 31.
//
// Every wait is bounded (2 s of wall time) and also gives up when another
// role has aborted; a wait that runs out writes status 1, every role stops
// issuing, waits (bounded) for what it issued, and the CTA frees its tensor
// memory and exits.

#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace mdr {

namespace {

constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kThreads = 192;

template <int BS, int D>
struct TcCfg {
  static constexpr bool kBig = (BS == 128 && D == 128);
  static constexpr int kQBuf = kBig ? 1 : 2;
  static constexpr int kStages = (BS == 64 && D == 64) ? 4 : 2;
  static constexpr int kPBuf = kBig ? 1 : 2;
  static constexpr int kTile = BS * D * 2;          // one [BS x D] bf16 tile
  static constexpr int kPBytes = BS * BS * 2;
  static constexpr int kRegion = BS * 128;          // one 64-column swizzled region of a tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBuf * kTile;
  static constexpr int kOffV = kOffK + kStages * kTile;
  static constexpr int kOffP = kOffV + kStages * kTile;
  static constexpr int kOffBar = kOffP + kPBuf * kPBytes;
  static constexpr int kOffMisc = kOffBar + 8 * 32;         // TMEM base address, abort flag
  static constexpr int kSmem = kOffMisc + 16;
  // M = 64 accumulators fill lanes 0-15 of each subpartition: two threads
  // share a row (16x32bx2 loads), each taking 32 of every 64 columns.
  static constexpr bool kHalf = (BS == 64);
  static constexpr int kSCols = kHalf ? 32 : BS;            // S columns per thread
  static constexpr int kColS = 0;                   // S buffers at columns 0 and BS
  static constexpr int kColO = 2 * BS;
  static constexpr int kCols = (2 * BS + D) <= 256 ? 256 : 512;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bQEmpty = bQFull + kQBuf;
  static constexpr int bKFull = bQEmpty + kQBuf;
  static constexpr int bKEmpty = bKFull + kStages;
  static constexpr int bVFull = bKEmpty + kStages;
  static constexpr int bVEmpty = bVFull + kStages;
  static constexpr int bSFull = bVEmpty + kStages;   // 2
  static constexpr int bPFull = bSFull + 2;          // kPBuf
  static constexpr int bPVDone = bPFull + kPBuf;     // 2
  static constexpr int bOFull = bPVDone + 2;
  static constexpr int bOFree = bOFull + 1;
  static constexpr int bFin = bOFree + 1;
  static constexpr int kNumBars = bFin + 1;
  static_assert(kNumBars <= 32, "barrier space");
  static_assert(kTile % 1024 == 0 && kPBytes % 1024 == 0, "1024-byte aligned tiles");
};

// Valid entries of a sel row are ids in [0, j]; everything else is skipped.
__device__ __forceinline__ bool valid_id(int id, int j) { return id >= 0 && id <= j; }

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  using namespace tc;
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > kWaitNs) return false;
  }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

}  // namespace

template <int BS, int D>
__global__ void __launch_bounds__(kThreads, BS == 64 ? 2 : 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const AttendArgs a) {
  using C = TcCfg<BS, D>;
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The swizzled tiles need 1024-byte alignment; the kernel declares no
  // static shared memory, so the dynamic region starts the CTA's window.
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(a.status, kDevMisaligned);
    return;
  }
  uint8_t* sm = smem_raw;
  uint32_t& tmem_base_s = *reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
  int& abort_s = *reinterpret_cast<int*>(sm + C::kOffMisc + 4);
  volatile int* abort_flag = &abort_s;
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t sQ = base + C::kOffQ, sK = base + C::kOffK, sV = base + C::kOffV, sP = base + C::kOffP;
  uint8_t* pP = sm + C::kOffP;
  const uint32_t bar0 = base + C::kOffBar;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = a.B * a.Hq * a.nb;
  const int g = a.Hq / a.Hkv;

  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), C::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kQBuf; ++i) { mbar_init(BAR(C::bQFull + i), 1); mbar_init(BAR(C::bQEmpty + i), 1); }
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(BAR(C::bKFull + i), 1);
      mbar_init(BAR(C::bKEmpty + i), 1);
      mbar_init(BAR(C::bVFull + i), 1);
      mbar_init(BAR(C::bVEmpty + i), 1);
    }
    for (int i = 0; i < 2; ++i) { mbar_init(BAR(C::bSFull + i), 1); mbar_init(BAR(C::bPVDone + i), 1); }
    for (int i = 0; i < C::kPBuf; ++i) mbar_init(BAR(C::bPFull + i), 4);
    mbar_init(BAR(C::bOFull), 1);
    mbar_init(BAR(C::bOFree), 4);
    mbar_init(BAR(C::bFin), 1);
    fence_mbar_init();
    abort_s = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  auto fail = [&]() {
    atomicExch(a.status, kDevWaitTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ----------------------------------------------------------- producers
    // Lane 0 loads Q and K, lane 1 loads V: a K stage is refilled as soon as
    // the S MMA that read it completes, independently of the later PV.
    if (lane < 2) {
      const bool is_k = lane == 0;
      if (is_k) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
      } else {
        prefetch_tmap(&tmV);
      }
      const int bFull = is_k ? C::bKFull : C::bVFull, bEmpty = is_k ? C::bKEmpty : C::bVEmpty;
      const uint32_t ring = is_k ? sK : sV;
      const void* tm = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
      int itv = 0, gb = 0;                      // non-empty tiles, blocks issued
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
        const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
        int nblk = 0;
        for (int e = 0; e < a.nsel; ++e) {
          const int id = row[e];
          if (valid_id(id, j)) ++nblk;
          else if (is_k && id >= 0) atomicExch(a.status, kDevBadSelection);
        }
        if (nblk == 0) continue;
        const int tok0 = b * a.S;
        if (is_k) {
          const int qs = itv % C::kQBuf;
          if (itv >= C::kQBuf && !wait_bar(BAR(C::bQEmpty + qs), ((itv / C::kQBuf) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(BAR(C::bQFull + qs), C::kTile);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)
            tma_load_3d(sQ + qs * C::kTile + gg * C::kRegion, &tmQ, BAR(C::bQFull + qs), gg * 64, hq,
                        tok0 + j * BS);
        }
        const int hkv = hq / g;
        for (int e = 0; e < a.nsel && ok; ++e) {
          const int id = row[e];
          if (!valid_id(id, j)) continue;
          const int st = gb % C::kStages;
          if (gb >= C::kStages && !wait_bar(BAR(bEmpty + st), ((gb / C::kStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(bFull + st);
          mbar_expect_tx(bar, C::kTile);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)
            tma_load_3d(ring + st * C::kTile + gg * C::kRegion, tm, bar, gg * 64, hkv, tok0 + id * BS);
          ++gb;
        }
        ++itv;
      }
      if (!ok) {
        fail();
        // Loads already issued: the last one of each stage completes after the
        // earlier ones of that stage.
        for (int st = 0; st < C::kStages; ++st) {
          int last = -1;
          for (int n = st; n < gb; n += C::kStages) last = n;
          if (last >= 0) mbar_wait(BAR(bFull + st), (last / C::kStages) & 1, kWaitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(BS, BS, 0, 0);
      const uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);
      const uint32_t tO = tmem + C::kColO;
      int itv = 0, g0 = 0;
      bool ok = true;
      auto issue_s = [&](int gblk, int qs) -> bool {
        const int st = gblk % C::kStages;
        if (!wait_bar(BAR(C::bKFull + st), (gblk / C::kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t tS = tmem + C::kColS + (gblk & 1) * BS;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kRegion + (kk % 4) * 32;
          mma_bf16(tS, smem_desc_sw128(sQ + qs * C::kTile + off, 16, 1024),
                   smem_desc_sw128(sK + st * C::kTile + off, 16, 1024), idS, kk > 0);
        }
        mma_commit(BAR(C::bSFull + (gblk & 1)));
        mma_commit(BAR(C::bKEmpty + st));
        return true;
      };
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int j = tile % a.nb;
        const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
        int nblk = 0;
        for (int e = 0; e < a.nsel; ++e) nblk += valid_id(row[e], j);
        if (nblk == 0) continue;
        const int qs = itv % C::kQBuf;
        if (!wait_bar(BAR(C::bQFull + qs), (itv / C::kQBuf) & 1, abort_flag)) { ok = false; break; }
        for (int n = 0; n < 2 && n < nblk && ok; ++n) ok = issue_s(g0 + n, qs);
        for (int n = 0; n < nblk && ok; ++n) {
          const int gblk = g0 + n;
          if (!wait_bar(BAR(C::bPFull + gblk % C::kPBuf), (gblk / C::kPBuf) & 1, abort_flag)) { ok = false; break; }
          if (n == 0 && itv > 0 && !wait_bar(BAR(C::bOFree), (itv - 1) & 1, abort_flag)) { ok = false; break; }
          if (!wait_bar(BAR(C::bVFull + gblk % C::kStages), (gblk / C::kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pbase = sP + (gblk % C::kPBuf) * C::kPBytes;
          const uint32_t vbase = sV + (gblk % C::kStages) * C::kTile;
#pragma unroll
          for (int kk = 0; kk < BS / 16; ++kk) {
            const uint32_t poff = (kk / 4) * C::kRegion + (kk % 4) * 32;
            mma_bf16(tO, smem_desc_sw128(pbase + poff, 16, 1024), smem_desc_sw128(vbase + kk * 2048, C::kRegion, 1024),
                     idPV, (n > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(BAR(C::bPVDone + (gblk & 1)));
          mma_commit(BAR(C::bVEmpty + gblk % C::kStages));
          if (n + 2 < nblk) ok = issue_s(gblk + 2, qs);
        }
        if (!ok) break;
        mma_commit(BAR(C::bQEmpty + qs));
        mma_commit(BAR(C::bOFull));
        g0 += nblk;
        ++itv;
      }
      if (!ok) fail();
      // Everything this thread issued has completed once bFin fires.
      mma_commit(BAR(C::bFin));
      mbar_wait(BAR(C::bFin), 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    constexpr bool kHalf = C::kHalf;
    constexpr int kSC = C::kSCols;
    const int sp = warp & 3;                          // TMEM subpartition of this warp
    const int hlf = kHalf ? (lane >> 4) : 0;          // M = 64: which 32 of each 64 columns
    const int r = kHalf ? (sp * 16 + (lane & 15)) : (sp * 32 + lane);
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    const uint32_t tO = tmem + C::kColO + lane_base;
    const float sl2 = a.scale * 1.4426950408889634f;  // scores in log2 units
    int itv = 0, g0 = 0;
    bool ok = true;
    // O chunk k of this thread: columns 64k + 32 hlf .. +31 (M = 64) or 32k .. +31.
    auto o_ld = [&](int k, float* o) {
      if constexpr (kHalf) tmem_ld16x2_32(tO + 64 * k, o);
      else tmem_ld32(tO + 32 * k, o);
    };
    auto o_st = [&](int k, const float* o) {
      if constexpr (kHalf) tmem_st16x2_32(tO + 64 * k, o);
      else tmem_st32(tO + 32 * k, o);
    };
    constexpr int kOChunks = kHalf ? D / 64 : D / 32;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
      const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
      int nblk = 0, diag = -1;
      for (int e = 0; e < a.nsel; ++e) {
        const int id = row[e];
        if (!valid_id(id, j)) continue;
        if (id == j) diag = nblk;
        ++nblk;
      }
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                           ((static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * BS + r) * a.Hq + hq) * D;
      if (nblk == 0) {                                 // nothing selected: zero output
        const int c_lo = kHalf ? hlf * (D / 16) : 0, c_hi = kHalf ? c_lo + D / 16 : D / 8;
        for (int c = c_lo; c < c_hi; ++c) reinterpret_cast<uint4*>(out)[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      float m_used = -INFINITY, l_sum = 0.f;
      for (int n = 0; n < nblk; ++n) {
        const int gblk = g0 + n;
        if (!wait_bar(BAR(C::bSFull + (gblk & 1)), (gblk >> 1) & 1, abort_flag)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        float sv[kSC];
        const uint32_t tS = tmem + C::kColS + (gblk & 1) * BS + lane_base;
        if constexpr (kHalf) {
          tmem_ld16x2_32(tS, sv);
        } else {
#pragma unroll
          for (int c = 0; c < BS / 32; ++c) tmem_ld32(tS + c * 32, sv + c * 32);
        }
        tmem_ld_wait();
        float mb = -INFINITY;
        const bool is_diag = n == diag;
        const int col0 = hlf * 32;
#pragma unroll
        for (int c = 0; c < kSC; ++c) {
          float x = sv[c] * sl2;
          if (is_diag && col0 + c > r) x = -INFINITY;
          sv[c] = x;
          mb = fmaxf(mb, x);
        }
        if constexpr (kHalf) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, 16));
        float alpha = 1.f;
        bool rescale = false;
        if (mb > m_used + 8.f) {
          alpha = exp2f(m_used - mb);
          rescale = n > 0;
          m_used = mb;
          l_sum *= alpha;
        }
        // O holds PV(n-1) once it completes; the P buffer is free once the PV
        // that last read it completed.
        const bool need_o = __any_sync(0xffffffffu, rescale);
        if (need_o && !wait_bar(BAR(C::bPVDone + ((gblk - 1) & 1)), ((gblk - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (gblk >= C::kPBuf &&
            !wait_bar(BAR(C::bPVDone + ((gblk - C::kPBuf) & 1)), ((gblk - C::kPBuf) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        if (need_o) {
          float o[32];
#pragma unroll
          for (int k = 0; k < kOChunks; ++k) {
            o_ld(k, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            o_st(k, o);
          }
          tmem_st_wait();
        }
        uint8_t* prow = pP + (gblk % C::kPBuf) * C::kPBytes + r * 128;
#pragma unroll
        for (int q = 0; q < kSC / 8; ++q) {
          const int q8 = hlf * 4 + q;                  // 8-column chunk of the row
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = exp2f(sv[q * 8 + e] - m_used);
            l_sum += p[e];
          }
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(p[2 * e], p[2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          const int region = q8 / 8, chunk = (q8 % 8) ^ (r % 8);
          *reinterpret_cast<uint4*>(prow + region * C::kRegion + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::bPFull + gblk % C::kPBuf));
      }
      if (!ok) break;
      // Epilogue: wait for the last PV of this tile, then O / sum -> bf16.
      if (!wait_bar(BAR(C::bOFull), itv & 1, abort_flag)) { ok = false; break; }
      __syncwarp();
      tc_fence_after();
      float l_row = l_sum;
      if constexpr (kHalf) l_row += __shfl_xor_sync(0xffffffffu, l_sum, 16);
      const float inv = 1.f / l_row;
#pragma unroll
      for (int k = 0; k < kOChunks; ++k) {
        float o[32];
        o_ld(k, o);
        tmem_ld_wait();
        const int col = kHalf ? 64 * k + 32 * hlf : 32 * k;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(o[q8 * 8 + 2 * e] * inv, o[q8 * 8 + 2 * e + 1] * inv);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(out + col + q8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bOFree));
      g0 += nblk;
      ++itv;
    }
    if (!ok) fail();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::kCols);
  }
}

namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  }
  return fn;
}

// [rows, H, D] bf16 viewed as a 3-D tensor (D, H, rows); box (64, 1, BS).
bool make_map(CUtensorMap* m, const void* ptr, long long rows, int H, int D, int BS) {
  EncodeTiled enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(BS)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BS, int D>
cudaError_t launch_tc(const AttendArgs& a, cudaStream_t st) {
  using C = TcCfg<BS, D>;
  CUtensorMap mq, mk, mv;
  const long long rows = static_cast<long long>(a.B) * a.S;
  if (!make_map(&mq, a.q, rows, a.Hq, D, BS) || !make_map(&mk, a.k, rows, a.Hkv, D, BS) ||
      !make_map(&mv, a.v, rows, a.Hkv, D, BS))
    return cudaErrorInvalidValue;
  auto k = attend_tc_kernel<BS, D>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, C::kSmem)) != cudaSuccess) return e;
  // Tensor memory: at most 512 columns per SM.
  per_sm = per_sm < 512 / C::kCols ? per_sm : 512 / C::kCols;
  if (per_sm < 1) per_sm = 1;
  const long long ntiles = static_cast<long long>(a.B) * a.Hq * a.nb;
  const long long want = static_cast<long long>(sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(ntiles < want ? ntiles : want);
  k<<<grid, kThreads, C::kSmem, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t st) {
  if (a.bs == 64 && a.D == 64) return launch_tc<64, 64>(a, st);
  if (a.bs == 64 && a.D == 128) return launch_tc<64, 128>(a, st);
  if (a.bs == 128 && a.D == 64) return launch_tc<128, 64>(a, st);
  if (a.bs == 128 && a.D == 128) return launch_tc<128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace mdr
