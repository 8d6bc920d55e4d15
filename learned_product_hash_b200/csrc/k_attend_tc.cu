// K5 (tensor cores): selected-set causal attention, bf16, on tcgen05 + TMEM.
//
// For token t of query block j and query head hq: softmax over every token s
// of the blocks listed in sel[b,hq,j] with s <= t of scale * <q'_t, k'_s>,
// applied to v_s ("Monodratic: a reproducible sparse attention mixer",
// section Mixer: exact causal softmax over the selected set, with the
// selected values themselves).
//
// Persistent, warp-specialised kernel, one CTA per SM.  A CTA walks the
// (b, hq, j) tiles blockIdx.x, blockIdx.x + gridDim.x, ... (consecutive CTAs
// take consecutive query blocks of one head, so that head's K/V stays in L2).
//   warp 0        TMA producers: lane 0 loads the Q tile of each query block
//                 into a Q ring and the K tile of every selected block into a
//                 K ring, lane 1 the V tiles into a V ring (128-byte swizzle,
//                 mbarrier expect-tx).  A K stage is refilled once the S MMA
//                 that read it completed, a V stage once its PV completed.
//   warp 1        MMA issuer (one lane).  The selected blocks of a tile are
//                 taken in groups of 128 keys: two consecutive 64-token
//                 blocks (their K tiles sit in adjacent stages of the K ring,
//                 which is laid out so that they form one 128-row operand),
//                 or one 128-token block.  S = Q K^T (M = bs, N = keys of
//                 the group, K = D) goes into one of two TMEM S buffers; O +=
//                 P V (M = bs, N = D, 16 keys per MMA, V read MN-major from
//                 its TMA tile) into one of two TMEM O accumulators,
//                 alternating by tile.  S of the next group is issued before
//                 the PV of the current one, across tile boundaries.  (A
//                 tcgen05.mma costs about 60 cycles however small it is, so
//                 wider N per instruction is what keeps the tensor pipe busy.)
//   warps 2..5    softmax: one query row per thread (two threads per row for
//                 bs = 64, whose accumulator rows fill lanes 0-15 of each
//                 subpartition: tcgen05.ld 16x32bx2), causal mask inside the
//                 query's own block, running maximum and sum in float32
//                 (log2 units, ex2.approx), P = exp(S - max) as bf16 into one
//                 of two shared-memory P buffers in the K-major 128-byte
//                 swizzled layout the PV MMA reads.  O is rescaled in TMEM only
//                 when the running maximum grows by more than 2^8 (exact, since
//                 the final division uses the same maximum).  A tile's epilogue
//                 (O / sum -> bf16 -> global) runs after the next tile's first
//                 P is handed over, overlapping tensor-core work.
// Warp w may only touch TMEM lanes 32 (w % 4) .. + 31.
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
constexpr int kThreads = 224;   // warp 0 K/Q producer, 1 MMA, 2-5 softmax, 6 V producer
constexpr int kSlots = 6;       // tile descriptors in flight
constexpr int kSlotInts = 68;   // tile, nblk, diag, 65 ids (nsel <= 64)

template <int BS, int D>
struct TcCfg {
  static constexpr bool kPair = (BS == 64);         // a group is two 64-token blocks
  static constexpr int kGroupKeys = 128;            // keys of a full group
  static constexpr bool kBig = (BS == 128 && D == 128);
  static constexpr int kQBuf = kBig ? 1 : 2;
  static constexpr int kKStages = (BS == 64) ? (D == 64 ? 8 : 6) : (D == 64 ? 4 : 2);   // even
  static constexpr int kVStages = (BS == 64) ? (D == 64 ? 8 : 4) : (D == 64 ? 4 : 2);
  static constexpr int kPBuf = kBig ? 1 : 2;
  static constexpr int kTile = BS * D * 2;          // one [BS x D] bf16 tile
  static constexpr int kRegion = BS * 128;          // 64 columns of one tile, 128B-swizzled
  static constexpr int kKRegion = kKStages * kRegion;   // K ring: region-major
  static constexpr int kPBytes = BS * kGroupKeys * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBuf * kTile;
  static constexpr int kOffV = kOffK + kKStages * kTile;
  static constexpr int kOffP = kOffV + kVStages * kTile;
  static constexpr int kOffBar = kOffP + kPBuf * kPBytes;
  static constexpr int kOffInfo = kOffBar + 8 * 64;         // tile descriptors
  static constexpr int kOffMisc = kOffInfo + kSlots * kSlotInts * 4;   // TMEM base, abort flag
  static constexpr int kSmem = kOffMisc + 16;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kKStages % 2 == 0, "pairs of K stages must not wrap");
  // bs = 64: two threads share an accumulator row (16x32bx2 loads).
  static constexpr bool kHalf = (BS == 64);
  // TMEM: two S buffers of 128 columns, two O accumulators of D columns.
  static constexpr int kColS = 0;
  static constexpr int kColO = 2 * kGroupKeys;
  static constexpr int kCols = (kColO + 2 * D) <= 256 ? 256 : 512;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bQEmpty = bQFull + kQBuf;
  static constexpr int bKFull = bQEmpty + kQBuf;
  static constexpr int bKEmpty = bKFull + kKStages;
  static constexpr int bVFull = bKEmpty + kKStages;
  static constexpr int bVEmpty = bVFull + kVStages;
  static constexpr int bSFull = bVEmpty + kVStages;  // 2
  static constexpr int bPFull = bSFull + 2;          // kPBuf
  static constexpr int bPVDone = bPFull + kPBuf;     // 2
  static constexpr int bOFull = bPVDone + 2;         // 2
  static constexpr int bOFree = bOFull + 2;          // 2
  static constexpr int bTFull = bOFree + 2;         // kSlots
  static constexpr int bTEmpty = bTFull + kSlots;    // kSlots
  static constexpr int bFin = bTEmpty + kSlots;
  static constexpr int kNumBars = bFin + 1;
  static_assert(kNumBars <= 64, "barrier space");
  static_assert(kTile % 1024 == 0 && kPBytes % 1024 == 0, "1024-byte aligned tiles");
};

// Valid entries of a sel row are ids in [0, j]; everything else is skipped.
__device__ __forceinline__ bool valid_id(int id, int j) { return id >= 0 && id <= j; }

// Size of the group that starts at global block g of a tile ending at gend.
template <bool kPair>
__device__ __forceinline__ int group_size(int g, int gend) {
  return (kPair && (g & 1) == 0 && g + 1 < gend) ? 2 : 1;
}

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

// 2^x on the special-function unit (ex2.approx.ftz: about 2 ulp, subnormal
// results flush to zero, which the softmax weights tolerate).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

}  // namespace

template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
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
  int32_t* info = reinterpret_cast<int32_t*>(sm + C::kOffInfo);   // [kSlots][kSlotInts]
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
    for (int i = 0; i < C::kKStages; ++i) { mbar_init(BAR(C::bKFull + i), 1); mbar_init(BAR(C::bKEmpty + i), 1); }
    for (int i = 0; i < C::kVStages; ++i) { mbar_init(BAR(C::bVFull + i), 1); mbar_init(BAR(C::bVEmpty + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::bSFull + i), 1);
      mbar_init(BAR(C::bPVDone + i), 1);
      mbar_init(BAR(C::bOFull + i), 1);
      mbar_init(BAR(C::bOFree + i), 4);
    }
    for (int i = 0; i < C::kPBuf; ++i) mbar_init(BAR(C::bPFull + i), 4);
    // A tile descriptor is released by the V producer, the MMA lane and the
    // four softmax warps.
    for (int i = 0; i < kSlots; ++i) { mbar_init(BAR(C::bTFull + i), 1); mbar_init(BAR(C::bTEmpty + i), 6); }
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
    // ------------------------------------------------ tile descriptors, Q, K
    // The warp reads each sel row once (lane e: entries e and e + 32),
    // compacts the valid ids with ballots into a shared-memory tile
    // descriptor for the other roles, then lane 0 loads Q and the K tiles.
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
    }
    int it = 0, itv = 0, gb = 0;               // tiles, non-empty tiles, blocks issued
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
      const int slot = it % kSlots;
      if (it >= kSlots && !wait_bar(BAR(C::bTEmpty + slot), ((it / kSlots) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
      const int e0 = lane < a.nsel ? row[lane] : -1, e1 = lane + 32 < a.nsel ? row[lane + 32] : -1;
      const bool v0 = valid_id(e0, j), v1 = valid_id(e1, j);
      if ((e0 >= 0 && !v0) || (e1 >= 0 && !v1)) atomicExch(a.status, kDevBadSelection);
      const unsigned m0 = __ballot_sync(0xffffffffu, v0), m1 = __ballot_sync(0xffffffffu, v1);
      const unsigned lt = (1u << lane) - 1u;
      int32_t* slot_p = info + slot * kSlotInts;
      if (v0) slot_p[3 + __popc(m0 & lt)] = e0;
      if (v1) slot_p[3 + __popc(m0) + __popc(m1 & lt)] = e1;
      const int nblk = __popc(m0) + __popc(m1);
      const unsigned d0 = __ballot_sync(0xffffffffu, v0 && e0 == j), d1 = __ballot_sync(0xffffffffu, v1 && e1 == j);
      if (lane == 0) {
        slot_p[0] = tile;
        slot_p[1] = nblk;
        slot_p[2] = d0 ? __popc(m0 & ((1u << (__ffs(d0) - 1)) - 1u))
                       : d1 ? __popc(m0) + __popc(m1 & ((1u << (__ffs(d1) - 1)) - 1u)) : -1;
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bTFull + slot));
      if (nblk == 0) continue;
      if (lane == 0) {
        const int tok0 = b * a.S;
        const int qs = itv % C::kQBuf;
        if (itv >= C::kQBuf && !wait_bar(BAR(C::bQEmpty + qs), ((itv / C::kQBuf) - 1) & 1, abort_flag)) ok = false;
        if (ok) {
          mbar_expect_tx(BAR(C::bQFull + qs), C::kTile);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)
            tma_load_3d(sQ + qs * C::kTile + gg * C::kRegion, &tmQ, BAR(C::bQFull + qs), gg * 64, hq,
                        tok0 + j * BS);
        }
        const int hkv = hq / g;
        for (int n = 0; n < nblk && ok; ++n) {
          const int id = slot_p[3 + n];
          const int st = gb % C::kKStages;
          if (gb >= C::kKStages &&
              !wait_bar(BAR(C::bKEmpty + st), ((gb / C::kKStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(C::bKFull + st);
          mbar_expect_tx(bar, C::kTile);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)   // region-major: region gg of every stage together
            tma_load_3d(sK + gg * C::kKRegion + st * C::kRegion, &tmK, bar, gg * 64, hkv, tok0 + id * BS);
          ++gb;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++itv;
    }
    if (!ok && lane == 0) {
      fail();
      for (int st = 0; st < C::kKStages; ++st) {
        int last = -1;
        for (int n = st; n < gb; n += C::kKStages) last = n;
        if (last >= 0) mbar_wait(BAR(C::bKFull + st), (last / C::kKStages) & 1, kWaitNs);
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      prefetch_tmap(&tmV);
      int it = 0, gb = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const int slot = it % kSlots;
        if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const int32_t* slot_p = info + slot * kSlotInts;
        const int nblk = slot_p[1];
        const int hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq), hkv = hq / g, tok0 = b * a.S;
        for (int n = 0; n < nblk && ok; ++n) {
          const int id = slot_p[3 + n];
          const int st = gb % C::kVStages;
          if (gb >= C::kVStages &&
              !wait_bar(BAR(C::bVEmpty + st), ((gb / C::kVStages) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(C::bVFull + st);
          mbar_expect_tx(bar, C::kTile);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)
            tma_load_3d(sV + st * C::kTile + gg * C::kRegion, &tmV, bar, gg * 64, hkv, tok0 + id * BS);
          ++gb;
        }
        if (ok) mbar_arrive(BAR(C::bTEmpty + slot));
      }
      if (!ok) {
        fail();
        for (int st = 0; st < C::kVStages; ++st) {
          int last = -1;
          for (int n = st; n < gb; n += C::kVStages) last = n;
          if (last >= 0) mbar_wait(BAR(C::bVFull + st), (last / C::kVStages) & 1, kWaitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS1 = idesc_bf16_f32(BS, BS, 0, 0);            // one block
      constexpr uint32_t idS2 = idesc_bf16_f32(BS, 2 * BS, 0, 0);        // a pair (bs = 64)
      constexpr uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);
      const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dP0 = smem_desc_sw128(sP, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sV, C::kRegion, 1024);
      constexpr uint32_t kTile16 = C::kTile / 16, kP16 = C::kPBytes / 16, kKReg16 = C::kKRegion / 16;
      constexpr uint32_t kRegion16 = C::kRegion / 16;
      // Tile queue: the PV cursor's tile and up to three after it, read from
      // the shared-memory tile descriptors (empty tiles are released at once).
      int q_nblk[4], q_g0[4], q_itv[4], q_slot[4];
      int nring = 0, head = 0;
      int next_it = 0, next_itv = 0, next_g0 = 0;
      const int my_tiles = blockIdx.x < ntiles ? (ntiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
      bool ok = true;
      // Append the next non-empty tile.  Only blocks when asked to: the
      // producer publishes a tile only after loading the previous tile's K,
      // which needs this lane's S MMAs.
      auto fetch = [&](bool block) {
        while (next_it < my_tiles && ok && nring < 4) {
          const int slot = next_it % kSlots;
          const uint32_t par = (next_it / kSlots) & 1;
          if (!block && !mbar_try_wait(BAR(C::bTFull + slot), par)) return;
          if (block && !wait_bar(BAR(C::bTFull + slot), par, abort_flag)) { ok = false; return; }
          ++next_it;
          const int nblk = info[slot * kSlotInts + 1];
          if (nblk == 0) { mbar_arrive(BAR(C::bTEmpty + slot)); continue; }
          const int qi = (head + nring) & 3;
#pragma unroll
          for (int x = 0; x < 4; ++x)
            if (x == qi) { q_nblk[x] = nblk; q_g0[x] = next_g0; q_itv[x] = next_itv; q_slot[x] = slot; }
          ++nring;
          next_g0 += nblk;
          ++next_itv;
          return;
        }
      };
      auto get = [&](const int* arr, int qi) {
        int v = arr[0];
#pragma unroll
        for (int x = 1; x < 4; ++x)
          if (x == qi) v = arr[x];
        return v;
      };
      int s_t = 0, s_b = -1;                     // S cursor: queue offset from head, next block (global)
      int Gs = 0, Gp = 0;                        // global group counters (S issued, PV issued)
      while (ok) {
        if (nring == 0) fetch(true);
        if (nring == 0) break;
        const int c_nblk = get(q_nblk, head), c_g0 = get(q_g0, head), c_itv = get(q_itv, head);
        const int c_end = c_g0 + c_nblk;
        const uint32_t tO = tmem + C::kColO + (c_itv & 1) * D;
        for (int gp = c_g0; gp < c_end && ok;) {
          const int np = group_size<C::kPair>(gp, c_end);
          // Issue S while at most one group ahead of this PV and at most one tile ahead.
          if (s_t >= nring - 1) fetch(false);
          while (Gs <= Gp + 1 && s_t < nring && s_t <= 1) {
            const int slot = (head + s_t) & 3;
            const int t_g0 = get(q_g0, slot), t_end = t_g0 + get(q_nblk, slot), t_itv = get(q_itv, slot);
            if (s_b < 0) s_b = t_g0;
            const int ns = group_size<C::kPair>(s_b, t_end);
            const int qs = t_itv % C::kQBuf;
            if (s_b == t_g0 && !wait_bar(BAR(C::bQFull + qs), (t_itv / C::kQBuf) & 1, abort_flag)) { ok = false; break; }
            const int st = s_b % C::kKStages;
            bool kready = wait_bar(BAR(C::bKFull + st), (s_b / C::kKStages) & 1, abort_flag);
            if (kready && ns == 2) kready = wait_bar(BAR(C::bKFull + st + 1), ((s_b + 1) / C::kKStages) & 1, abort_flag);
            if (!kready) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = tmem + C::kColS + (Gs & 1) * C::kGroupKeys;
            const uint64_t dq = dQ0 + qs * kTile16, dk = dK0 + st * kRegion16;
            const uint32_t idS = ns == 2 ? idS2 : idS1;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qoff = ((kk / 4) * C::kRegion + (kk % 4) * 32) / 16;
              const uint32_t koff = (kk / 4) * kKReg16 + (kk % 4) * 2;
              if (kk == 0) mma_bf16_c<false>(tS, dq + qoff, dk + koff, idS);
              else mma_bf16_c<true>(tS, dq + qoff, dk + koff, idS);
            }
            mma_commit(BAR(C::bSFull + (Gs & 1)));
            mma_commit(BAR(C::bKEmpty + st));
            if (ns == 2) mma_commit(BAR(C::bKEmpty + st + 1));
            ++Gs;
            s_b += ns;
            if (s_b == t_end) {                   // all S of that tile issued: its Q slot frees
              mma_commit(BAR(C::bQEmpty + qs));
              s_b = -1;
              ++s_t;
              if (s_t >= nring) fetch(false);
            }
          }
          if (!ok) break;
          // PV of group Gp (blocks gp .. gp + np - 1).
          if (!wait_bar(BAR(C::bPFull + Gp % C::kPBuf), (Gp / C::kPBuf) & 1, abort_flag)) { ok = false; break; }
          if (gp == c_g0 && c_itv >= 2 &&
              !wait_bar(BAR(C::bOFree + (c_itv & 1)), ((c_itv >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dp = dP0 + (Gp % C::kPBuf) * kP16;
          for (int h = 0; h < np && ok; ++h) {
            const int blk = gp + h, vs = blk % C::kVStages;
            if (!wait_bar(BAR(C::bVFull + vs), (blk / C::kVStages) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t dv = dV0 + vs * kTile16;
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
              // keys 16kk.. of this block: P region (h*BS + 16kk)/64, V rows 16kk..
              const int key = h * BS + kk * 16;
              const uint32_t poff = ((key / 64) * C::kRegion + ((key % 64) / 16) * 32) / 16;
              if (kk == 0 && h == 0 && gp == c_g0) mma_bf16_c<false>(tO, dp + poff, dv + kk * 128, idPV);
              else mma_bf16_c<true>(tO, dp + poff, dv + kk * 128, idPV);
            }
            mma_commit(BAR(C::bVEmpty + vs));
          }
          if (!ok) break;
          mma_commit(BAR(C::bPVDone + (Gp & 1)));
          ++Gp;
          gp += np;
        }
        if (!ok) break;
        mma_commit(BAR(C::bOFull + (c_itv & 1)));
        mbar_arrive(BAR(C::bTEmpty + get(q_slot, head)));
        head = (head + 1) & 3;
        --nring;
        --s_t;
      }
      if (!ok) fail();
      // Everything this thread issued has completed once bFin fires.
      mma_commit(BAR(C::bFin));
      mbar_wait(BAR(C::bFin), 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    constexpr bool kHalf = C::kHalf;
    // Columns of a group held by this thread: bs = 64: 64 (32 of each block);
    // bs = 128: 128.
    constexpr int kSC = kHalf ? 64 : 128;
    const int sp = warp & 3;                          // TMEM subpartition of this warp
    const int hlf = kHalf ? (lane >> 4) : 0;          // bs = 64: which 32 of each 64 columns
    const int r = kHalf ? (sp * 16 + (lane & 15)) : (sp * 32 + lane);
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    const float sl2 = a.scale * 1.4426950408889634f;  // scores in log2 units
    constexpr int kOChunks = kHalf ? D / 64 : D / 32;
    // O chunk k of this thread: columns 64k + 32 hlf .. +31 (bs = 64) or 32k .. +31.
    auto o_ld = [&](uint32_t tO, int k, float* o) {
      if constexpr (kHalf) tmem_ld16x2_32(tO + 64 * k, o);
      else tmem_ld32(tO + 32 * k, o);
    };
    auto o_st = [&](uint32_t tO, int k, const float* o) {
      if constexpr (kHalf) tmem_st16x2_32(tO + 64 * k, o);
      else tmem_st32(tO + 32 * k, o);
    };
    bool pend = false;
    int pend_itv = 0;
    float pend_l = 1.f;
    __nv_bfloat16* pend_out = nullptr;
    auto epilogue = [&]() -> bool {
      if (!wait_bar(BAR(C::bOFull + (pend_itv & 1)), (pend_itv >> 1) & 1, abort_flag)) return false;
      __syncwarp();
      tc_fence_after();
      const uint32_t tO = tmem + C::kColO + (pend_itv & 1) * D + lane_base;
      const float inv = 1.f / pend_l;
#pragma unroll
      for (int k = 0; k < kOChunks; ++k) {
        float o[32];
        o_ld(tO, k, o);
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
          *reinterpret_cast<uint4*>(pend_out + col + q8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bOFree + (pend_itv & 1)));
      pend = false;
      return true;
    };
    int it = 0, itv = 0, g0 = 0, G = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
      const int slot = it % kSlots;
      if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
      const int nblk = info[slot * kSlotInts + 1], diag = info[slot * kSlotInts + 2];
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bTEmpty + slot));
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                           ((static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * BS + r) * a.Hq + hq) * D;
      if (nblk == 0) {                                 // nothing selected: zero output
        const int c_lo = kHalf ? hlf * (D / 16) : 0, c_hi = kHalf ? c_lo + D / 16 : D / 8;
        for (int c = c_lo; c < c_hi; ++c) reinterpret_cast<uint4*>(out)[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const uint32_t tO = tmem + C::kColO + (itv & 1) * D + lane_base;
      const int gend = g0 + nblk;
      float m_used = -INFINITY, l_sum = 0.f;          // running max in log2 units
      bool first = true;
      for (int gb = g0; gb < gend; ++G) {
        const int ng = group_size<C::kPair>(gb, gend);
        const int n_in_tile = gb - g0;              // index of the group's first block in the tile
        if (!wait_bar(BAR(C::bSFull + (G & 1)), (G >> 1) & 1, abort_flag)) { ok = false; break; }
        __syncwarp();
        tc_fence_after();
        float sv[kSC];
        const uint32_t tS = tmem + C::kColS + (G & 1) * C::kGroupKeys + lane_base;
        if constexpr (kHalf) {
          tmem_ld16x2_32(tS, sv);                  // block 0 of the group
          if (ng == 2) tmem_ld16x2_32(tS + 64, sv + 32);
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv + c * 32);
        }
        tmem_ld_wait();
        // Column c of sv: block c / 32 of the group, key 32 hlf + c % 32 (bs = 64);
        // block 0, key c (bs = 128).
        constexpr int kPerBlk = kHalf ? 32 : 128;
        const int nvalid = kHalf ? 32 * ng : 128;
#pragma unroll
        for (int c = 0; c < kSC; ++c) {
          const int blk = c / kPerBlk, key = (kHalf ? 32 * hlf : 0) + c % kPerBlk;
          if (c >= nvalid || (n_in_tile + blk == diag && key > r)) sv[c] = -INFINITY;
        }
        float mraw = -INFINITY;
#pragma unroll
        for (int c = 0; c < kSC; ++c) mraw = fmaxf(mraw, sv[c]);
        if constexpr (kHalf) mraw = fmaxf(mraw, __shfl_xor_sync(0xffffffffu, mraw, 16));
        const float mb = mraw * sl2;
        float alpha = 1.f;
        bool rescale = false;
        if (mb > m_used + 8.f) {
          alpha = ex2_approx(m_used - mb);
          rescale = !first;
          m_used = mb;
          l_sum *= alpha;
        }
        // O holds PV(G-1) once it completes; the P buffer is free once the PV
        // that last read it completed.
        const bool need_o = __any_sync(0xffffffffu, rescale);
        if (need_o && !wait_bar(BAR(C::bPVDone + ((G - 1) & 1)), ((G - 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (G >= C::kPBuf &&
            !wait_bar(BAR(C::bPVDone + ((G - C::kPBuf) & 1)), ((G - C::kPBuf) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        if (need_o) {
          float o[32];
#pragma unroll
          for (int k = 0; k < kOChunks; ++k) {
            o_ld(tO, k, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            o_st(tO, k, o);
          }
          tmem_st_wait();
        }
        uint8_t* prow = pP + (G % C::kPBuf) * C::kPBytes + r * 128;
#pragma unroll
        for (int q = 0; q < kSC / 8; ++q) {
          // 8 columns of sv -> group key kq .. kq+7
          const int blk = (q * 8) / kPerBlk;
          const int kq = blk * BS + (kHalf ? 32 * hlf : 0) + (q * 8) % kPerBlk;
          if (kHalf && blk >= ng) break;
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2_approx(__fmaf_rn(sv[q * 8 + e], sl2, -m_used));
            l_sum += p[e];
          }
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat162 h = __floats2bfloat162_rn(p[2 * e], p[2 * e + 1]);
            w[e] = *reinterpret_cast<uint32_t*>(&h);
          }
          const int region = kq / 64, chunk = ((kq % 64) / 8) ^ (r % 8);
          *reinterpret_cast<uint4*>(prow + region * C::kRegion + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::bPFull + G % C::kPBuf));
        if (first && pend && !epilogue()) { ok = false; break; }
        first = false;
        gb += ng;
      }
      if (!ok) break;
      float l_row = l_sum;
      if constexpr (kHalf) l_row += __shfl_xor_sync(0xffffffffu, l_sum, 16);
      pend = true;
      pend_itv = itv;
      pend_l = l_row;
      pend_out = out;
      g0 = gend;
      ++itv;
    }
    if (ok && pend && !epilogue()) ok = false;
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
