// K5 (tensor cores): selected-set causal attention, bf16, on tcgen05 + TMEM.
//
// For token t of query block j and query head hq: softmax over every token s
// of the blocks listed in sel[b,hq,j] with s <= t of scale * <q'_t, k'_s>,
// applied to v_s ("Monodratic: a reproducible sparse attention mixer",
// section Mixer: exact causal softmax over the selected set, with the
// selected values themselves).
//
// Persistent, warp-specialised kernel, one CTA per SM.  The CTAs take
// (b, hq, j) tiles from a global counter, head by head and within a head from
// the last query block down: the CTAs running at any time work on
// neighbouring query blocks of one head (that head's K/V stays in L2), and
// the last tiles handed out are the first query blocks, which select the
// fewest blocks, so the CTAs finish close together.
// The selected blocks of a tile are taken in groups of 128 keys: two
// consecutive 64-token blocks, or one 128-token block.
//   warp 0        reads each sel row once (warp-parallel, ballot compaction)
//                 into a shared-memory ring of tile descriptors, then lane 0
//                 loads the Q tile and each group's K tiles by TMA into a
//                 ring of group slots (laid out so that a group's two K tiles
//                 form one 128-row, 128-byte-swizzled operand).
//   warp 10       loads each group's V tiles into a second ring of slots.
//   warp 1        MMA issuer (one lane): S = Q K^T (M = bs, N = keys of the
//                 group, K = D) into one of two TMEM S buffers, O += P V (M =
//                 bs, N = D, 16 keys per MMA, V read MN-major from its TMA
//                 tile) into one of two TMEM O accumulators, alternating by
//                 tile.  S of the next group is issued before the PV of the
//                 current one, across tile boundaries.  One full/empty
//                 mbarrier pair per group slot keeps waits and commits at a
//                 few per group (each costs tens of cycles; a tcgen05.mma
//                 about 60 however small it is).
//   warps 2..9    softmax, two warps per TMEM subpartition, each taking 64 of
//                 a group's 128 columns: rows of the accumulator (two threads
//                 per row for bs = 64, whose rows fill lanes 0-15 of each
//                 subpartition: tcgen05.ld 16x32bx2), causal mask inside the
//                 query's own block, the row maximum exchanged between the two
//                 warps through shared memory and a named barrier, running
//                 maximum and sum in float32 (log2 units, ex2.approx), P =
//                 exp(S - max) as bf16 into one of two shared-memory P buffers
//                 in the K-major swizzled layout the PV MMA reads.  O is
//                 rescaled in TMEM only when the running maximum grows by more
//                 than 2^8 (exact: the final division uses the same maximum).
//                 A tile's epilogue (O / sum -> bf16 -> global) runs after the
//                 next tile's first P is handed over, overlapping MMA work.
// Warp w may only touch TMEM lanes 32 (w % 4) .. + 31.
//
// Every wait is bounded (2 s of wall time) and also gives up when another
// role has aborted; a wait that runs out writes status 1, every role stops
// issuing, waits (bounded) for what it issued, and the CTA frees its tensor
// memory and exits.

#include <cuda.h>

#include "attend_tc_common.cuh"
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tmap.h"

namespace mdr {

namespace {

using atc::kWaitNs;
using atc::valid_id;
using atc::wait_bar;
using atc::ex2_approx;
using atc::pack_bf16;
constexpr int kThreads = 352;   // 11 warps
constexpr int kSlots = 4;       // tile descriptors in flight
constexpr int kSlotBytes = 144; // int32 tile; int16 nblk, diag; int16 ids[64]

template <int BS, int D>
struct TcCfg {
  static constexpr bool kPair = (BS == 64);         // a group is two 64-token blocks
  static constexpr int kGroupKeys = 128;
  static constexpr bool kBig = (BS == 128 && D == 128);
  static constexpr int kQBuf = kBig ? 1 : 2;
  static constexpr int kKSlots = (BS == 64) ? (D == 64 ? 4 : 3) : (D == 64 ? 3 : 2);
  static constexpr int kVSlots = (BS == 64) ? (D == 64 ? 4 : 2) : (D == 64 ? 3 : 2);
  static constexpr int kPBuf = kBig ? 1 : 2;
  static constexpr int kTile = BS * D * 2;          // one [BS x D] bf16 block tile
  static constexpr int kGroupBytes = kGroupKeys * D * 2;
  static constexpr int kRegion = BS * 128;          // 64 columns of one block tile
  static constexpr int kGRegion = kGroupKeys * 128; // 64 columns of one group slot
  static constexpr int kKRing = kKSlots * kGRegion; // K ring: region-major
  static constexpr int kPBytes = BS * kGroupKeys * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBuf * kTile;
  static constexpr int kOffV = kOffK + kKSlots * kGroupBytes;
  static constexpr int kOffP = kOffV + kVSlots * kGroupBytes;
  static constexpr int kOffBar = kOffP + kPBuf * kPBytes;
  static constexpr int kNumBarsMax = 48;
  static constexpr int kOffInfo = kOffBar + 8 * kNumBarsMax;
  static constexpr int kOffXch = kOffInfo + kSlots * kSlotBytes;       // [2][2][BS] row maxima
  static constexpr int kOffXl = kOffXch + 2 * 2 * BS * 4;             // [2][BS] row sums
  static constexpr int kOffMisc = kOffXl + 2 * BS * 4;                 // TMEM base, abort flag
  static constexpr int kSmem = kOffMisc + 16;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static constexpr bool kHalfRows = (BS == 64);     // two threads per accumulator row
  // TMEM: two S buffers of 128 columns, two O accumulators of D columns.
  static constexpr int kColS = 0;
  static constexpr int kColO = 2 * kGroupKeys;
  static constexpr int kCols = (kColO + 2 * D) <= 256 ? 256 : 512;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bQEmpty = bQFull + kQBuf;
  static constexpr int bKFull = bQEmpty + kQBuf;
  static constexpr int bKEmpty = bKFull + kKSlots;
  static constexpr int bVFull = bKEmpty + kKSlots;
  static constexpr int bVEmpty = bVFull + kVSlots;
  static constexpr int bSFull = bVEmpty + kVSlots;   // 2
  static constexpr int bPFull = bSFull + 2;          // kPBuf (8 arrivals)
  static constexpr int bPVDone = bPFull + kPBuf;     // 2
  static constexpr int bOFull = bPVDone + 2;         // 2
  static constexpr int bOFree = bOFull + 2;          // 2 (8 arrivals)
  static constexpr int bTFull = bOFree + 2;          // kSlots
  static constexpr int bTEmpty = bTFull + kSlots;    // kSlots (10 arrivals)
  static constexpr int bX = bTEmpty + kSlots;       // 4 (2 arrivals): row exchange per subpartition
  static constexpr int bFin = bX + 4;
  static constexpr int kNumBars = bFin + 1;
  static_assert(kNumBars <= kNumBarsMax, "barrier space");
  static_assert(kTile % 1024 == 0 && kPBytes % 1024 == 0 && kGRegion % 1024 == 0, "1024-byte aligned tiles");
};

// Size of the group that starts at block n (0-based, in the tile's list) of
// a tile with nblk selected blocks: blocks 0-1, 2-3, ... pair up for bs = 64.
template <bool kPair>
__device__ __forceinline__ int group_size(int n, int nblk) {
  return (kPair && (n & 1) == 0 && n + 1 < nblk) ? 2 : 1;
}

}  // namespace

// kLse: also write each row's softmax normaliser (a separate instantiation,
// so that the plain forward carries none of it).
template <int BS, int D, bool kLse>
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
  uint8_t* info = sm + C::kOffInfo;
  float* xch = reinterpret_cast<float*>(sm + C::kOffXch);   // [G & 1][half][row]
  float* xl = reinterpret_cast<float*>(sm + C::kOffXl);     // [half][row]
  const uint32_t bar0 = base + C::kOffBar;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  auto slot_tile = [&](int s) -> int& { return *reinterpret_cast<int*>(info + s * kSlotBytes); };
  auto slot_s16 = [&](int s, int i) -> int16_t& { return *reinterpret_cast<int16_t*>(info + s * kSlotBytes + 4 + 2 * i); };
  // slot_s16(s, 0) = nblk, (s, 1) = diag, (s, 2 + n) = id n

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;         // query blocks a.j0 .. a.j0 + nbr - 1
  const int ntiles = a.B * a.Hq * nbr;
  const int g = a.Hq / a.Hkv;

  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_base_s), C::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kQBuf; ++i) { mbar_init(BAR(C::bQFull + i), 1); mbar_init(BAR(C::bQEmpty + i), 1); }
    for (int i = 0; i < C::kKSlots; ++i) { mbar_init(BAR(C::bKFull + i), 1); mbar_init(BAR(C::bKEmpty + i), 1); }
    for (int i = 0; i < C::kVSlots; ++i) { mbar_init(BAR(C::bVFull + i), 1); mbar_init(BAR(C::bVEmpty + i), 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(BAR(C::bSFull + i), 1);
      mbar_init(BAR(C::bPVDone + i), 1);
      mbar_init(BAR(C::bOFull + i), 1);
      mbar_init(BAR(C::bOFree + i), 8);
    }
    for (int i = 0; i < C::kPBuf; ++i) mbar_init(BAR(C::bPFull + i), 8);
    // A tile descriptor is released by the V producer, the MMA lane and the
    // eight softmax warps.
    for (int i = 0; i < kSlots; ++i) { mbar_init(BAR(C::bTFull + i), 1); mbar_init(BAR(C::bTEmpty + i), 10); }
    for (int i = 0; i < 4; ++i) mbar_init(BAR(C::bX + i), 2);
    mbar_init(BAR(C::bFin), 1);
    fence_mbar_init();
    abort_s = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;
  grid_dependency_wait();          // q', k' and sel come from earlier kernels

  auto fail = [&]() {
    atomicExch(a.status, kDevWaitTimeout);
    *abort_flag = 1;
  };

  if (warp == 0) {
    // ------------------------------------------------ tile descriptors, Q, K
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
    }
    int itv = 0, G = 0;                        // non-empty tiles, groups issued
    int last_q[2] = {-1, -1};                  // last tile whose Q each buffer received
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (it >= kSlots &&
          !__all_sync(0xffffffffu, wait_bar(BAR(C::bTEmpty + slot), ((it / kSlots) - 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      int t = 0;
      if (lane == 0) t = atomicAdd(a.tile_counter, 1);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (t >= ntiles) {                       // no tiles left: tile -1 ends every role's loop
        if (lane == 0) {
          slot_tile(slot) = -1;
          __threadfence_block();
          mbar_arrive(BAR(C::bTFull + slot));
        }
        break;
      }
      const int tile = (t / nbr) * a.nb + (a.j0 + nbr - 1 - t % nbr);
      const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
      const int32_t* row = a.sel + static_cast<size_t>(tile) * a.nsel;
      const int e0 = lane < a.nsel ? row[lane] : -1, e1 = lane + 32 < a.nsel ? row[lane + 32] : -1;
      const bool v0 = valid_id(e0, j), v1 = valid_id(e1, j);
      if ((e0 >= 0 && !v0) || (e1 >= 0 && !v1)) atomicExch(a.status, kDevBadSelection);
      const unsigned m0 = __ballot_sync(0xffffffffu, v0), m1 = __ballot_sync(0xffffffffu, v1);
      const unsigned lt = (1u << lane) - 1u;
      if (v0) slot_s16(slot, 2 + __popc(m0 & lt)) = static_cast<int16_t>(e0);
      if (v1) slot_s16(slot, 2 + __popc(m0) + __popc(m1 & lt)) = static_cast<int16_t>(e1);
      const int nblk = __popc(m0) + __popc(m1);
      const unsigned d0 = __ballot_sync(0xffffffffu, v0 && e0 == j), d1 = __ballot_sync(0xffffffffu, v1 && e1 == j);
      if (lane == 0) {
        slot_tile(slot) = tile;
        slot_s16(slot, 0) = static_cast<int16_t>(nblk);
        slot_s16(slot, 1) = static_cast<int16_t>(
            d0 ? __popc(m0 & ((1u << (__ffs(d0) - 1)) - 1u))
               : d1 ? __popc(m0) + __popc(m1 & ((1u << (__ffs(d1) - 1)) - 1u)) : -1);
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
          last_q[qs] = itv;
        }
        const int hkv = hq / g;
        for (int n = 0; n < nblk && ok; ++G) {
          const int ng = group_size<C::kPair>(n, nblk);
          const int ks = G % C::kKSlots;
          if (G >= C::kKSlots && !wait_bar(BAR(C::bKEmpty + ks), ((G / C::kKSlots) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(C::bKFull + ks);
          mbar_expect_tx(bar, ng * C::kTile);
          for (int h = 0; h < ng; ++h) {
            const int id = slot_s16(slot, 2 + n + h);
#pragma unroll
            for (int gg = 0; gg < D / 64; ++gg)
              tma_load_3d(sK + gg * C::kKRing + ks * C::kGRegion + h * C::kRegion, &tmK, bar, gg * 64, hkv,
                          tok0 + id * BS);
          }
          n += ng;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++itv;
    }
    if (!ok && lane == 0) {
      fail();
      for (int k = 0; k < C::kKSlots; ++k) {
        int last = -1;
        for (int n = k; n < G; n += C::kKSlots) last = n;
        if (last >= 0) mbar_wait(BAR(C::bKFull + k), (last / C::kKSlots) & 1, kWaitNs);
      }
      for (int k = 0; k < C::kQBuf; ++k)
        if (last_q[k] >= 0) mbar_wait(BAR(C::bQFull + k), (last_q[k] / C::kQBuf) & 1, kWaitNs);
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      prefetch_tmap(&tmV);
      int G = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const int tile = slot_tile(slot);
        if (tile < 0) break;
        const int nblk = slot_s16(slot, 0);
        const int hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq), hkv = hq / g, tok0 = b * a.S;
        for (int n = 0; n < nblk && ok; ++G) {
          const int ng = group_size<C::kPair>(n, nblk);
          const int vs = G % C::kVSlots;
          if (G >= C::kVSlots && !wait_bar(BAR(C::bVEmpty + vs), ((G / C::kVSlots) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(C::bVFull + vs);
          mbar_expect_tx(bar, ng * C::kTile);
          for (int h = 0; h < ng; ++h) {
            const int id = slot_s16(slot, 2 + n + h);
#pragma unroll
            for (int gg = 0; gg < D / 64; ++gg)
              tma_load_3d(sV + vs * C::kGroupBytes + h * C::kTile + gg * C::kRegion, &tmV, bar, gg * 64, hkv,
                          tok0 + id * BS);
          }
          n += ng;
        }
        if (ok) mbar_arrive(BAR(C::bTEmpty + slot));
      }
      if (!ok) {
        fail();
        for (int k = 0; k < C::kVSlots; ++k) {
          int last = -1;
          for (int n = k; n < G; n += C::kVSlots) last = n;
          if (last >= 0) mbar_wait(BAR(C::bVFull + k), (last / C::kVSlots) & 1, kWaitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS1 = idesc_bf16_f32(BS, BS, 0, 0);            // one block
      constexpr uint32_t idS2 = idesc_bf16_f32(BS, C::kPair ? 2 * BS : BS, 0, 0);   // a pair
      constexpr uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);
      const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dP0 = smem_desc_sw128(sP, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sV, C::kRegion, 1024);
      // Tile queue: the PV cursor's tile and up to three after it.
      int q_nblk[4], q_g0[4], q_itv[4];
      int nring = 0, head = 0;
      int next_it = 0, next_itv = 0, next_g0 = 0;
      bool ok = true, tiles_left = true;
      auto get = [&](const int* arr, int qi) {
        int v = arr[0];
#pragma unroll
        for (int x = 1; x < 4; ++x)
          if (x == qi) v = arr[x];
        return v;
      };
      // Append the next non-empty tile.  Only blocks when asked to: the
      // producer publishes a tile only after loading the previous tile's K,
      // which needs this lane's S MMAs.
      auto fetch = [&](bool block) {
        while (tiles_left && ok && nring < 4) {
          const int slot = next_it % kSlots;
          const uint32_t par = (next_it / kSlots) & 1;
          if (!block && !mbar_try_wait(BAR(C::bTFull + slot), par)) return;
          if (block && !wait_bar(BAR(C::bTFull + slot), par, abort_flag)) { ok = false; return; }
          if (slot_tile(slot) < 0) { tiles_left = false; return; }
          ++next_it;
          const int nblk = slot_s16(slot, 0);
          mbar_arrive(BAR(C::bTEmpty + slot));   // nothing else is read from the slot
          if (nblk == 0) continue;
          const int qi = (head + nring) & 3;
#pragma unroll
          for (int x = 0; x < 4; ++x)
            if (x == qi) { q_nblk[x] = nblk; q_g0[x] = next_g0; q_itv[x] = next_itv; }
          ++nring;
          next_g0 += nblk;
          ++next_itv;
          return;
        }
      };
      int s_t = 0, s_b = -1;                     // S cursor: queue offset from head, next block (global)
      int Gs = 0, Gp = 0;                        // groups whose S / PV were issued
      while (ok) {
        if (nring == 0) fetch(true);
        if (nring == 0) break;
        const int c_g0 = get(q_g0, head), c_end = c_g0 + get(q_nblk, head), c_itv = get(q_itv, head);
        const uint32_t tO = tmem + C::kColO + (c_itv & 1) * D;
        for (int gp = c_g0; gp < c_end && ok;) {
          const int np = group_size<C::kPair>(gp - c_g0, c_end - c_g0);
          // Issue S while at most one group ahead of this PV and one tile ahead.
          if (s_t >= nring - 1) fetch(false);
          while (Gs <= Gp + 1 && s_t < nring && s_t <= 1) {
            const int qi = (head + s_t) & 3;
            const int t_g0 = get(q_g0, qi), t_end = t_g0 + get(q_nblk, qi), t_itv = get(q_itv, qi);
            if (s_b < 0) s_b = t_g0;
            const int ns = group_size<C::kPair>(s_b - t_g0, t_end - t_g0);
            const int qs = t_itv % C::kQBuf, ks = Gs % C::kKSlots;
            if (s_b == t_g0 && !wait_bar(BAR(C::bQFull + qs), (t_itv / C::kQBuf) & 1, abort_flag)) { ok = false; break; }
            if (!wait_bar(BAR(C::bKFull + ks), (Gs / C::kKSlots) & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tS = tmem + C::kColS + (Gs & 1) * C::kGroupKeys;
            const uint64_t dq = dQ0 + qs * (C::kTile / 16), dk = dK0 + ks * (C::kGRegion / 16);
            const uint32_t idS = ns == 2 ? idS2 : idS1;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t qoff = ((kk / 4) * C::kRegion + (kk % 4) * 32) / 16;
              const uint32_t koff = (kk / 4) * (C::kKRing / 16) + (kk % 4) * 2;
              if (kk == 0) mma_bf16_c<false>(tS, dq + qoff, dk + koff, idS);
              else mma_bf16_c<true>(tS, dq + qoff, dk + koff, idS);
            }
            mma_commit(BAR(C::bSFull + (Gs & 1)));
            mma_commit(BAR(C::bKEmpty + ks));
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
          const int vs = Gp % C::kVSlots;
          if (!wait_bar(BAR(C::bPFull + Gp % C::kPBuf), (Gp / C::kPBuf) & 1, abort_flag)) { ok = false; break; }
          if (gp == c_g0 && c_itv >= 2 &&
              !wait_bar(BAR(C::bOFree + (c_itv & 1)), ((c_itv >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          if (!wait_bar(BAR(C::bVFull + vs), (Gp / C::kVSlots) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dp = dP0 + (Gp % C::kPBuf) * (C::kPBytes / 16);
          for (int h = 0; h < np; ++h) {
            const uint64_t dv = dV0 + vs * (C::kGroupBytes / 16) + h * (C::kTile / 16);
#pragma unroll
            for (int kk = 0; kk < BS / 16; ++kk) {
              const int key = h * BS + kk * 16;   // P region key / 64, V rows 16 kk ..
              const uint32_t poff = ((key / 64) * C::kRegion + ((key % 64) / 16) * 32) / 16;
              if (kk == 0 && h == 0 && gp == c_g0) mma_bf16_c<false>(tO, dp + poff, dv + kk * 128, idPV);
              else mma_bf16_c<true>(tO, dp + poff, dv + kk * 128, idPV);
            }
          }
          mma_commit(BAR(C::bPVDone + (Gp & 1)));
          mma_commit(BAR(C::bVEmpty + vs));
          ++Gp;
          gp += np;
        }
        if (!ok) break;
        mma_commit(BAR(C::bOFull + (c_itv & 1)));
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
    constexpr bool kHR = C::kHalfRows;
    constexpr int kSC = kHR ? 32 : 64;                // S columns per thread per group
    const int sp = warp & 3;                          // TMEM subpartition
    const int half = (warp - 2) >> 2;                 // which 64 of a group's 128 columns
    const int tsub = kHR ? (lane >> 4) : 0;           // bs = 64: which 32 of those 64
    const int r = kHR ? (sp * 16 + (lane & 15)) : (sp * 32 + lane);
    const bool writer = !kHR || tsub == 0;            // one lane per row publishes row values
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    // Waits give the same answer in every lane (a lane may see the abort flag
    // while another already saw the phase complete).
    auto wwait = [&](int bar, uint32_t par) {
      return __all_sync(0xffffffffu, wait_bar(BAR(bar), par, abort_flag));
    };
    // Row values pass between the two warps of a subpartition through shared
    // memory; each exchange is one phase of that pair's mbarrier.
    int xph = 0;
    auto exchange = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bX + sp));
      const bool done = wwait(C::bX + sp, xph & 1);
      ++xph;
      return done;
    };
    const float sl2 = a.scale * 1.4426950408889634f;  // scores in log2 units
    // This thread's O columns: kHR: (D/2) half + (D/4) tsub, D/4 of them (one
    // 16x32bx2 load); otherwise (D/2) half + 32 i for i < D/64.
    constexpr int kOParts = kHR ? 1 : D / 64;
    constexpr int kOW = kHR ? D / 4 : 32;
    auto o_col = [&](int i) { return (D / 2) * half + (kHR ? (D / 4) * tsub : 32 * i); };
    auto o_ld = [&](uint32_t tO, int i, float* o) {
      if constexpr (kHR) {
        if constexpr (D == 128) tmem_ld16x2_32(tO + (D / 2) * half, o);
        else tmem_ld16x2_16(tO + (D / 2) * half, o);
      } else {
        tmem_ld32(tO + (D / 2) * half + 32 * i, o);
      }
    };
    auto o_st = [&](uint32_t tO, int i, const float* o) {
      if constexpr (kHR) {
        if constexpr (D == 128) tmem_st16x2_32(tO + (D / 2) * half, o);
        else tmem_st16x2_16(tO + (D / 2) * half, o);
      } else {
        tmem_st32(tO + (D / 2) * half + 32 * i, o);
      }
    };
    bool pend = false;
    int pend_itv = 0;
    float pend_l = 0.f, pend_m = 0.f;
    __nv_bfloat16* pend_out = nullptr;
    float* pend_lse = nullptr;                       // this row's normaliser, when asked for
    auto epilogue = [&]() -> bool {
      if (!wwait(C::bOFull + (pend_itv & 1), (pend_itv >> 1) & 1)) return false;
      // Row sum: the two threads of a row, then the partner warp.
      float l = pend_l;
      if constexpr (kHR) l += __shfl_xor_sync(0xffffffffu, l, 16);
      if (writer) xl[half * BS + r] = l;
      if (!exchange()) return false;
      l += xl[(1 - half) * BS + r];
      if constexpr (kLse)
        if (writer && half == 0) *pend_lse = (pend_m + __log2f(l)) * 0.6931471805599453f;
      tc_fence_after();
      const uint32_t tO = tmem + C::kColO + (pend_itv & 1) * D + lane_base;
      const float inv = 1.f / l;
#pragma unroll
      for (int i = 0; i < kOParts; ++i) {
        float o[kOW];
        o_ld(tO, i, o);
        tmem_ld_wait();
#pragma unroll
        for (int q8 = 0; q8 < kOW / 8; ++q8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) w[e] = pack_bf16(o[q8 * 8 + 2 * e] * inv, o[q8 * 8 + 2 * e + 1] * inv);
          *reinterpret_cast<uint4*>(pend_out + o_col(i) + q8 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bOFree + (pend_itv & 1)));
      pend = false;
      return true;
    };
    int itv = 0, g0 = 0, G = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (!wwait(C::bTFull + slot, (it / kSlots) & 1)) { ok = false; break; }
      const int tile = slot_tile(slot), nblk = slot_s16(slot, 0), diag = slot_s16(slot, 1);
      if (tile < 0) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bTEmpty + slot));
      const int j = tile % a.nb, hq = (tile / a.nb) % a.Hq, b = tile / (a.nb * a.Hq);
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                           ((static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * BS + r) * a.Hq + hq) * D;
      float* lse = kLse ? a.lse + (static_cast<size_t>(b) * a.Hq + hq) * a.S + static_cast<size_t>(j) * BS + r : nullptr;
      if (nblk == 0) {                                 // nothing selected: zero output
        for (int i = 0; i < kOParts; ++i)
          for (int q8 = 0; q8 < kOW / 8; ++q8) *reinterpret_cast<uint4*>(out + o_col(i) + q8 * 8) = make_uint4(0, 0, 0, 0);
        if constexpr (kLse)
          if (writer && half == 0) *lse = -INFINITY;
        continue;
      }
      const uint32_t tO = tmem + C::kColO + (itv & 1) * D + lane_base;
      const int gend = g0 + nblk;
      float m_used = -INFINITY, l_sum = 0.f;          // running max in log2 units
      bool first = true;
      for (int gb = g0; gb < gend; ++G) {
        const int n_in_tile = gb - g0;
        const int ng = group_size<C::kPair>(n_in_tile, nblk);
        const bool has = !C::kPair || half < ng;      // bs = 64: the second block of a pair
        if (!wwait(C::bSFull + (G & 1), (G >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        float sv[kSC];
        float pmax = -INFINITY;
        if (has) {
          const uint32_t tS = tmem + C::kColS + (G & 1) * C::kGroupKeys + lane_base + 64 * half;
          if constexpr (kHR) {
            tmem_ld16x2_32(tS, sv);
          } else {
            tmem_ld32(tS, sv);
            tmem_ld32(tS + 32, sv + 32);
          }
          tmem_ld_wait();
          // Column c: block (kPair ? half : 0) of the group, key kb + c.
          const int blk = C::kPair ? half : 0;
          const int kb = kHR ? 32 * tsub : 64 * half;
          if (n_in_tile + blk == diag) {
#pragma unroll
            for (int c = 0; c < kSC; ++c)
              if (kb + c > r) sv[c] = -INFINITY;
          }
#pragma unroll
          for (int c = 0; c < kSC; ++c) pmax = fmaxf(pmax, sv[c]);
        }
        if constexpr (kHR) pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, 16));
        float* xg = xch + (G & 1) * 2 * BS;
        if (writer) xg[half * BS + r] = pmax;
        if (!exchange()) { ok = false; break; }
        const float mb = fmaxf(pmax, xg[(1 - half) * BS + r]) * sl2;
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
        if (need_o && !wwait(C::bPVDone + ((G - 1) & 1), ((G - 1) >> 1) & 1)) {
          ok = false;
          break;
        }
        if (G >= C::kPBuf &&
            !wwait(C::bPVDone + ((G - C::kPBuf) & 1), ((G - C::kPBuf) >> 1) & 1)) {
          ok = false;
          break;
        }
        __syncwarp();
        tc_fence_after();
        if (need_o) {
          float o[kOW];
#pragma unroll
          for (int i = 0; i < kOParts; ++i) {
            o_ld(tO, i, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < kOW; ++e) o[e] *= alpha;
            o_st(tO, i, o);
          }
          tmem_st_wait();
        }
        if (has) {
          // P region `half` holds keys 64 half .. of the group; this thread's
          // 8-key chunks start at chunk (kHR ? 4 tsub : 0).
          uint8_t* prow = pP + (G % C::kPBuf) * C::kPBytes + half * C::kRegion + r * 128;
#pragma unroll
          for (int q = 0; q < kSC / 8; ++q) {
            float p[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              p[e] = ex2_approx(__fmaf_rn(sv[q * 8 + e], sl2, -m_used));
              l_sum += p[e];
            }
            const int chunk = ((kHR ? 4 * tsub : 0) + q) ^ (r % 8);
            *reinterpret_cast<uint4*>(prow + chunk * 16) =
                make_uint4(pack_bf16(p[0], p[1]), pack_bf16(p[2], p[3]), pack_bf16(p[4], p[5]), pack_bf16(p[6], p[7]));
          }
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
      pend = true;
      pend_itv = itv;
      pend_l = l_sum;
      pend_m = m_used;
      pend_out = out;
      pend_lse = lse;
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

template <int BS, int D>
cudaError_t launch_tc(const AttendArgs& a, cudaStream_t st) {
  using C = TcCfg<BS, D>;
  CUtensorMap mq, mk, mv;
  const long long rows = static_cast<long long>(a.B) * a.S;
  if (!make_tile_map(&mq, a.q, rows, a.Hq, D, BS) || !make_tile_map(&mk, a.k, rows, a.Hkv, D, BS) ||
      !make_tile_map(&mv, a.v, rows, a.Hkv, D, BS))
    return cudaErrorInvalidValue;
  auto k = a.lse ? attend_tc_kernel<BS, D, true> : attend_tc_kernel<BS, D, false>;
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(k), C::kSmem);
  if (e != cudaSuccess) return e;
  const int sms = cached_sm_count();
  int per_sm = cached_occupancy(reinterpret_cast<const void*>(k), kThreads, C::kSmem);
  if (sms <= 0) return cudaErrorUnknown;
  // Tensor memory: at most 512 columns per SM.
  per_sm = per_sm < 512 / C::kCols ? per_sm : 512 / C::kCols;
  if (per_sm < 1) per_sm = 1;
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return cudaErrorInvalidValue;
  const long long ntiles = static_cast<long long>(a.B) * a.Hq * nbr;
  const long long want = static_cast<long long>(sms) * per_sm;
  const unsigned grid = static_cast<unsigned>(ntiles < want ? ntiles : want);
  // Every CTA takes one tile number past the last: the counter reaches ntiles + grid.
  if (!a.tile_counter || ntiles + grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  e = launch_pdl(k, dim3(grid), dim3(kThreads), C::kSmem, st, mq, mk, mv, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t st) {
  if (a.bs == 128 && a.Hkv > 0 && a.Hq / a.Hkv >= 2) return launch_attend_union(a, st);
  if (a.bs == 64 && a.D == 64) return launch_tc<64, 64>(a, st);
  if (a.bs == 64 && a.D == 128) return launch_tc<64, 128>(a, st);
  if (a.bs == 128 && a.D == 64) return launch_tc<128, 64>(a, st);
  if (a.bs == 128 && a.D == 128) return launch_tc<128, 128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace mdr
