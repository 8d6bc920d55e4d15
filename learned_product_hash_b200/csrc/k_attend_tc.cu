// K5 (tensor cores): selected-set causal attention, bf16, on tcgen05 + TMEM.
//
// For token t of query block j and query head hq: softmax over every token s
// of the blocks listed in sel[b,hq,j] with s <= t of scale * <q'_t, k'_s>,
// applied to v_s ("Monodratic: a reproducible sparse attention mixer",
// section Mixer: exact causal softmax over the selected set, with the
// selected values themselves).
//
// One CTA (4 warps) per (b, hq, j).  Thread 0 drives the asynchronous units:
// TMA brings the Q tile and, block by block, the K and V tiles of the
// selected blocks into a two-stage ring of 128-byte-swizzled shared memory;
// tcgen05.mma computes S = Q K^T (M = bs query rows, N = bs keys, K = D) into
// tensor memory and O += P V (M = bs, N = D, K = bs keys) into a second TMEM
// accumulator.  All 128 threads run the softmax: each owns one query row of
// S (tcgen05.ld), applies the causal mask inside the query's own block,
// keeps a running maximum and sum in float32, writes P = exp(S - max) as
// bf16 into shared memory in the layout the next MMA reads, and rescales O
// in TMEM only when the running maximum grows by more than 2^8 (exact:
// the final division by the running sum uses the same maximum).
//
// Tensor-memory layout of an accumulator with M = 64: row r sits in lane
// (r % 16) + 32 * (r / 16); with M = 128 row r sits in lane r.  Warp w reads
// lanes 32w..32w+31.
//
// Every mbarrier wait is bounded (2 s of wall time).  A wait that runs out
// writes kDevWaitTimeout to the status word, the CTA stops issuing work,
// waits (bounded) for what it already issued, frees its tensor memory and
// exits.

#include <cuda.h>

#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace mdr {

namespace {

constexpr uint64_t kWaitNs = 2000000000ull;

template <int BS, int D>
struct TcCfg {
  static constexpr int kStages = 2;
  static constexpr int kTileBytes = BS * D * 2;     // one [BS x D] bf16 tile
  static constexpr int kPBytes = BS * BS * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffP = kOffV + kStages * kTileBytes;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr int kSmem = kOffBar + 128 + 1024;  // barriers + alignment slack
  static constexpr int kColS = 0;
  static constexpr int kColO = BS;
  static constexpr int kCols = (BS + D) <= 128 ? 128 : 256;
  static constexpr int kRegion = BS * 128;            // one 64-column swizzled region of a tile
  static_assert(kTileBytes % 1024 == 0 && kPBytes % 1024 == 0, "1024-byte aligned tiles");
};

enum Bar { kBarQ = 0, kBarKV = 1, kBarFree = 3, kBarS = 5, kBarDone = 6 };

}  // namespace

template <int BS, int D>
__global__ void __launch_bounds__(128, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const AttendArgs a) {
  using C = TcCfg<BS, D>;
  using namespace tc;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_base_s;
  __shared__ int blocks[kMaxSel];
  __shared__ int nblk_s;
  __shared__ int abort_s;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* sm = smem_raw + (base - raw);
  const uint32_t sQ = base + C::kOffQ, sK = base + C::kOffK, sV = base + C::kOffV, sP = base + C::kOffP;
  uint8_t* pP = sm + C::kOffP;
  const uint32_t bar0 = base + C::kOffBar;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int j = tile % a.nb;
  const int hq = (tile / a.nb) % a.Hq;
  const int b = tile / (a.nb * a.Hq);
  const int hkv = hq / (a.Hq / a.Hkv);

  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_base_s), C::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < 7; ++i) mbar_init(BAR(i), 1);
    fence_mbar_init();
    abort_s = 0;
  }
  if (threadIdx.x == 64) {
    const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
    int n = 0;
    for (int e = 0; e < a.nsel; ++e) {
      const int id = row[e];
      if (id < 0) continue;
      if (id > j || id >= a.nb) { atomicExch(a.status, kDevBadSelection); continue; }
      blocks[n++] = id;
    }
    nblk_s = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  const uint32_t tS = tmem + C::kColS, tO = tmem + C::kColO;
  const int nblk = nblk_s;
  const int tok0 = b * a.S;                   // first token row of sequence b

  if (nblk == 0) {                            // nothing selected: the output is zero
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
    for (int e = threadIdx.x; e < BS * D / 8; e += blockDim.x) {
      const int rr = e / (D / 8), c8 = e % (D / 8);
      *reinterpret_cast<uint4*>(out + ((static_cast<size_t>(tok0) + static_cast<size_t>(j) * BS + rr) * a.Hq + hq) * D +
                                c8 * 8) = make_uint4(0, 0, 0, 0);
    }
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    if (warp == 0) tmem_dealloc(tmem, C::kCols);
    return;
  }

  const uint32_t idS = idesc_bf16_f32(BS, BS, 0, 0);
  const uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);
  int issued = 0;                             // K/V blocks whose TMA thread 0 issued

  auto issue_kv = [&](int n, int s) {
    const uint32_t bar = BAR(kBarKV + s);
    mbar_expect_tx(bar, 2 * C::kTileBytes);
    const int row = tok0 + blocks[n] * BS;
#pragma unroll
    for (int g = 0; g < D / 64; ++g) {
      tma_load_3d(sK + s * C::kTileBytes + g * C::kRegion, &tmK, bar, g * 64, hkv, row);
      tma_load_3d(sV + s * C::kTileBytes + g * C::kRegion, &tmV, bar, g * 64, hkv, row);
    }
  };
  auto issue_s = [&](int s) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = (kk / 4) * C::kRegion + (kk % 4) * 32;
      mma_bf16(tS, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK + s * C::kTileBytes + off, 16, 1024),
               idS, kk > 0);
    }
    mma_commit(BAR(kBarS));
  };
  auto fail = [&]() {
    atomicExch(a.status, kDevWaitTimeout);
    abort_s = 1;
  };

  bool t0_fail = false;
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    mbar_expect_tx(BAR(kBarQ), C::kTileBytes);
#pragma unroll
    for (int g = 0; g < D / 64; ++g) tma_load_3d(sQ + g * C::kRegion, &tmQ, BAR(kBarQ), g * 64, hq, tok0 + j * BS);
    for (int n = 0; n < C::kStages && n < nblk; ++n) { issue_kv(n, n); ++issued; }
    if (mbar_wait(BAR(kBarQ), 0, kWaitNs) && mbar_wait(BAR(kBarKV), 0, kWaitNs)) {
      tc_fence_after();
      issue_s(0);
    } else {
      t0_fail = true;
      fail();
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(BAR(kBarS)) : "memory");
    }
  }

  const bool has_row = (BS == 128) || (lane < 16);
  const int r = (BS == 128) ? (warp * 32 + lane) : (warp * 16 + lane);
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  const float sl2 = a.scale * 1.4426950408889634f;   // scores in log2 units
  float m_used = -INFINITY, l_sum = 0.f;
  bool aborted = false;

  for (int n = 0; n < nblk; ++n) {
    const int s = n % C::kStages;
    bool bad = !mbar_wait(BAR(kBarS), n & 1, kWaitNs);
    __syncwarp();                               // tcgen05.ld is warp-collective
    tc_fence_after();
    float sv[BS];
#pragma unroll
    for (int c = 0; c < BS / 32; ++c) tmem_ld32(tS + lane_base + c * 32, sv + c * 32);
    tmem_ld_wait();
    float alpha = 1.f;
    bool rescale = false;
    if (has_row) {
      const bool diag = blocks[n] == j;
      float mb = -INFINITY;
#pragma unroll
      for (int c = 0; c < BS; ++c) {
        float x = sv[c] * sl2;
        if (diag && c > r) x = -INFINITY;
        sv[c] = x;
        mb = fmaxf(mb, x);
      }
      if (mb > m_used + 8.f) {
        alpha = exp2f(m_used - mb);
        rescale = n > 0;
        m_used = mb;
        l_sum *= alpha;
      }
      uint8_t* prow = pP + r * 128;
#pragma unroll
      for (int q8 = 0; q8 < BS / 8; ++q8) {
        float p[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          p[e] = exp2f(sv[q8 * 8 + e] - m_used);
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
    }
    __syncwarp();
    if (__any_sync(0xffffffffu, rescale)) {
      float o[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(tO + lane_base + c * 32, o);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] *= alpha;
        tmem_st32(tO + lane_base + c * 32, o);
      }
      tmem_st_wait();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    if (__syncthreads_or(bad || t0_fail || abort_s)) {
      aborted = true;
      if (bad && threadIdx.x == 0) fail();
      break;
    }
    if (threadIdx.x == 0) {
      tc_fence_after();
      const uint32_t vbase = sV + s * C::kTileBytes;
#pragma unroll
      for (int kk = 0; kk < BS / 16; ++kk) {
        const uint32_t poff = (kk / 4) * C::kRegion + (kk % 4) * 32;
        mma_bf16(tO, smem_desc_sw128(sP + poff, 16, 1024), smem_desc_sw128(vbase + kk * 2048, C::kRegion, 1024),
                 idPV, (n > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(BAR(kBarFree + s));
      if (n + 1 < nblk) {
        const int s1 = (n + 1) % C::kStages;
        if (mbar_wait(BAR(kBarKV + s1), ((n + 1) / C::kStages) & 1, kWaitNs)) {
          tc_fence_after();
          issue_s(s1);
        } else {
          t0_fail = true;
          fail();
          asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(BAR(kBarS)) : "memory");
        }
      }
      if (!t0_fail && n + C::kStages < nblk) {
        if (mbar_wait(BAR(kBarFree + s), (n / C::kStages) & 1, kWaitNs)) {
          issue_kv(n + C::kStages, s);
          ++issued;
        } else {
          t0_fail = true;
          fail();
        }
      }
    }
  }

  // Drain: every MMA this CTA issued, and every TMA still in flight.
  if (threadIdx.x == 0) {
    tc_fence_after();
    mma_commit(BAR(kBarDone));
    if (aborted || t0_fail) {
      // The last load issued into each stage completes after the earlier ones.
      for (int s = 0; s < C::kStages; ++s) {
        int last = -1;
        for (int n = s; n < issued; n += C::kStages) last = n;
        if (last >= 0) mbar_wait(BAR(kBarKV + s), (last / C::kStages) & 1, kWaitNs);
      }
      mbar_wait(BAR(kBarQ), 0, kWaitNs);
    }
  }
  const bool done = mbar_wait(BAR(kBarDone), 0, kWaitNs);
  __syncwarp();
  if (!done && threadIdx.x == 0) fail();
  tc_fence_after();
  if (done && !aborted && !__syncthreads_or(abort_s)) {
    const float inv = 1.f / l_sum;
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                         ((static_cast<size_t>(tok0) + static_cast<size_t>(j) * BS + r) * a.Hq + hq) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      tmem_ld32(tO + lane_base + c * 32, o);
      tmem_ld_wait();
      if (has_row) {
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(o[q8 * 8 + 2 * e] * inv, o[q8 * 8 + 2 * e + 1] * inv);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(out + c * 32 + q8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  __syncwarp();
  if (warp == 0) tmem_dealloc(tmem, C::kCols);
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
  const unsigned grid = static_cast<unsigned>(a.B) * a.Hq * a.nb;
  k<<<grid, 128, C::kSmem, st>>>(mq, mk, mv, a);
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
