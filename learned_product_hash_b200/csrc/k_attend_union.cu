// K5u (tensor cores, grouped query heads, 128-token blocks): selected-set
// causal attention that gathers each selected key block once for a pair of
// query heads.
//
// Result as in the one-head-per-tile kernel (k_attend_tc.cu): for token t of
// query block j and query head hq, softmax over the tokens s <= t of the
// blocks listed in sel[b,hq,j] of scale * <q'_t, k'_s>, applied to v_s
// ("Monodratic: a reproducible sparse attention mixer", section Mixer: exact
// causal softmax over the selected set).  A block listed twice in one row
// counts once: the row is a set.
//
// The query heads of a KV-head group largely select the same key blocks
// (their block means route through the same product codes), and the
// attention is bound by the bytes each SM takes in from the memory system
// (about 46 GB/s per SM for TMA tile loads on B200, L2 hits or not).  So the
// unit of work here is a pair of query heads (hq, hq + 1) of one KV head at
// one query block j: the union of the two rows' blocks is gathered once, and
// each block's K and V tiles serve both heads where both selected it.
//   warp 0     reads the two sel rows, builds their union (ascending ids, a
//              two-bit membership mask per id) into a shared-memory ring of
//              unit descriptors, then loads the unit's Q tiles and each union
//              block's K tile by TMA.
//   warp 10    loads each union block's V tile.
//   warp 1     MMA issuer (one lane).  A unit is a sequence of steps, one per
//              (union block, head that selected it).  Step n: S = Q_h K^T
//              (M = 128 query rows, N = 128 keys, K = D) into TMEM S buffer
//              n % 2; O_h += P V with P read from tensor memory -- the softmax
//              writes P as bf16 pairs over the S buffer it came from -- and V
//              MN-major from its TMA tile.  S of step n + 1 is issued before
//              the PV of step n; S of step n + 2 waits for the PV of step n
//              to complete (it overwrites that step's P).
//   warps 2-9  softmax, two warps per TMEM subpartition, 64 of the 128 key
//              columns each; the row maximum is exchanged between the two
//              through shared memory; running maximum and sum per head in
//              float32 (log2 units); O rescaled in TMEM only when the maximum
//              grows by more than 2^8.  A unit's two outputs are written after
//              the next unit's first P is handed over.
// TMEM: two S buffers (128 columns each), then O of the two heads (D columns
// each): 512 columns, one CTA per SM.  Units are taken from a global counter,
// pair by pair and within a pair from the last query block down.
//
// Every wait is bounded (2 s of wall time) and gives up when another role
// has aborted; a wait that runs out writes status 1, every role stops
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

using atc::ex2_approx;
using atc::kWaitNs;
using atc::pack_bf16;
using atc::valid_id;
using atc::wait_bar;

constexpr int kThreads = 384;      // 12 warps
constexpr int kSlots = 4;          // unit descriptors in flight
constexpr int kMaxU = 128;         // union of two rows of at most 64 entries
// Unit descriptor: int32 unit; int16 nA, nB, nu, diag; int16 ids[kMaxU];
// uint8 mask[kMaxU] (bit 0: the first head selected the block, bit 1: the
// second).
constexpr int kUIds = 12;
constexpr int kUMask = kUIds + 2 * kMaxU;
constexpr int kSlotBytes = 400;
static_assert(kUMask + kMaxU <= kSlotBytes, "unit descriptor");

template <int D>
struct UCfg {
  static constexpr int BS = 128;
  static constexpr int kTile = BS * D * 2;            // one [128 x D] bf16 tile
  static constexpr int kRegion = BS * 128;            // 64 columns of a tile
  static constexpr int kQBuf = (D == 128) ? 1 : 2;    // Q tile pairs
  static constexpr int kKSlots = (D == 128) ? 2 : 4;
  static constexpr int kVSlots = (D == 128) ? 2 : 4;
  static constexpr int kKRing = kKSlots * kRegion;    // K ring: region-major
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBuf * 2 * kTile;
  static constexpr int kOffV = kOffK + kKSlots * kTile;
  static constexpr int kOffBar = kOffV + kVSlots * kTile;
  static constexpr int kNumBarsMax = 48;
  static constexpr int kOffInfo = kOffBar + 8 * kNumBarsMax;
  static constexpr int kOffScr = kOffInfo + kSlots * kSlotBytes;  // int16 ids[kMaxU], uint8 first[kMaxU]
  static constexpr int kOffXch = kOffScr + 3 * kMaxU;             // [2][2][BS] row maxima
  static constexpr int kOffXl = kOffXch + 2 * 2 * BS * 4;         // [2 heads][2][BS] row sums
  static constexpr int kOffStage = kOffXl + 2 * 2 * BS * 4;       // per softmax warp: 2 KB output staging
  static constexpr int kOffMisc = kOffStage + 8 * 2048;           // TMEM base, abort flag
  static constexpr int kSmem = kOffMisc + 16;
  static_assert(kSmem <= 232448, "shared memory per CTA");
  static_assert(kTile % 1024 == 0 && kRegion % 1024 == 0, "1024-byte aligned tiles");
  // TMEM columns
  static constexpr int kColS = 0;                     // S buffer b at 128 b; P over its first 64
  static constexpr int kColO = 256;                   // O of head x at kColO + D x
  static constexpr int kCols = 512;
  // barrier indices
  static constexpr int bQFull = 0;
  static constexpr int bQEmpty = bQFull + kQBuf;
  static constexpr int bKFull = bQEmpty + kQBuf;
  static constexpr int bKEmpty = bKFull + kKSlots;
  static constexpr int bVFull = bKEmpty + kKSlots;
  static constexpr int bVEmpty = bVFull + kVSlots;
  static constexpr int bSFull = bVEmpty + kVSlots;    // 2
  static constexpr int bPFull = bSFull + 2;           // 2 (8 arrivals)
  static constexpr int bPVDone = bPFull + 2;          // 2
  static constexpr int bOFull = bPVDone + 2;          // 1
  static constexpr int bOFree = bOFull + 1;           // 1 (8 arrivals)
  static constexpr int bTFull = bOFree + 1;           // kSlots
  static constexpr int bTEmpty = bTFull + kSlots;     // kSlots (10 arrivals)
  static constexpr int bX = bTEmpty + kSlots;         // 4 (2 arrivals): row exchange per subpartition
  static constexpr int bFin = bX + 4;
  static constexpr int kNumBars = bFin + 1;
  static_assert(kNumBars <= kNumBarsMax, "barrier space");
};

// One step of a unit as the MMA lane queues it between S and PV.
struct Step {
  int slot, x, vg, itv;
  bool first_entry, last_entry, first_unit, first_x, last_unit;
};

}  // namespace

// kLse: also write each row's softmax normaliser (a separate instantiation).
template <int D, bool kLse>
__global__ void __launch_bounds__(kThreads, 1)
attend_union_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttendArgs a) {
  using C = UCfg<D>;
  constexpr int BS = C::BS;
  using namespace tc;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(a.status, kDevMisaligned);
    return;
  }
  uint8_t* sm = smem_raw;
  uint32_t& tmem_base_s = *reinterpret_cast<uint32_t*>(sm + C::kOffMisc);
  int& abort_s = *reinterpret_cast<int*>(sm + C::kOffMisc + 4);
  volatile int* abort_flag = &abort_s;
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t sQ = base + C::kOffQ, sK = base + C::kOffK, sV = base + C::kOffV;
  uint8_t* info = sm + C::kOffInfo;
  float* xch = reinterpret_cast<float*>(sm + C::kOffXch);   // [step & 1][half][row]
  float* xl = reinterpret_cast<float*>(sm + C::kOffXl);     // [head][half][row]
  const uint32_t bar0 = base + C::kOffBar;
  auto BAR = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  auto u_unit = [&](int s) -> int& { return *reinterpret_cast<int*>(info + s * kSlotBytes); };
  auto u_hdr = [&](int s, int i) -> int16_t& { return *reinterpret_cast<int16_t*>(info + s * kSlotBytes + 4 + 2 * i); };
  auto u_id = [&](int s, int e) -> int16_t& { return *reinterpret_cast<int16_t*>(info + s * kSlotBytes + kUIds + 2 * e); };
  auto u_mask = [&](int s, int e) -> uint8_t& { return *(info + s * kSlotBytes + kUMask + e); };
  // u_hdr(s, 0) = nA, (s, 1) = nB, (s, 2) = nu, (s, 3) = diag (union position of block j, or -1)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = a.Hq / a.Hkv;
  const int npair = (g + 1) / 2;
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;         // query blocks a.j0 .. a.j0 + nbr - 1
  const int nunits = a.B * a.Hkv * npair * nbr;

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
      mbar_init(BAR(C::bPFull + i), 8);
      mbar_init(BAR(C::bPVDone + i), 1);
    }
    mbar_init(BAR(C::bOFull), 1);
    mbar_init(BAR(C::bOFree), 8);
    // A unit descriptor is released by the Q/K and V producers, the MMA lane
    // and the eight softmax warps.
    for (int i = 0; i < kSlots; ++i) { mbar_init(BAR(C::bTFull + i), 1); mbar_init(BAR(C::bTEmpty + i), 11); }
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
  // Unit t -> (b, hkv, pair p, j): pairs in order, query blocks from the last.
  auto decode = [&](int t, int& b, int& hkv, int& p, int& j) {
    const int bp = t / nbr;
    j = a.j0 + nbr - 1 - (t - bp * nbr);
    p = bp % npair;
    const int bh = bp / npair;
    hkv = bh % a.Hkv;
    b = bh / a.Hkv;
  };

  if (warp == 11) {
    // ---------------------------------------------------- unit descriptors
    int16_t* scr_id = reinterpret_cast<int16_t*>(sm + C::kOffScr);   // valid ids, first row's then second's
    uint8_t* scr_first = sm + C::kOffScr + 2 * kMaxU;                // 1 where an id occurs first
    const unsigned lt = (1u << lane) - 1u;
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
      if (t >= nunits) {                       // no units left: unit -1 ends every role's loop
        if (lane == 0) {
          u_unit(slot) = -1;
          __threadfence_block();
          mbar_arrive(BAR(C::bTFull + slot));
        }
        break;
      }
      int b, hkv, p, j;
      decode(t, b, hkv, p, j);
      const int hqA = hkv * g + 2 * p;
      const bool hasB = 2 * p + 1 < g;
      const int32_t* rowA = a.sel + (static_cast<size_t>(b) * a.Hq + hqA) * a.nb * a.nsel + static_cast<size_t>(j) * a.nsel;
      const int32_t* rowB = rowA + static_cast<size_t>(a.nb) * a.nsel;   // head hqA + 1, same block
      int ev[4];
      ev[0] = lane < a.nsel ? rowA[lane] : -1;
      ev[1] = lane + 32 < a.nsel ? rowA[lane + 32] : -1;
      ev[2] = hasB && lane < a.nsel ? rowB[lane] : -1;
      ev[3] = hasB && lane + 32 < a.nsel ? rowB[lane + 32] : -1;
      bool vv[4];
      unsigned mm[4];
      bool bad = false;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        vv[k] = valid_id(ev[k], j);
        bad |= ev[k] >= 0 && !vv[k];
        mm[k] = __ballot_sync(0xffffffffu, vv[k]);
      }
      if (bad) atomicExch(a.status, kDevBadSelection);
      const int nA = __popc(mm[0]) + __popc(mm[1]), nB = __popc(mm[2]) + __popc(mm[3]);
      const int nall = nA + nB;
      __syncwarp();                            // the previous unit's reads of the scratch are done
      const int pos[4] = {__popc(mm[0] & lt), __popc(mm[0]) + __popc(mm[1] & lt), nA + __popc(mm[2] & lt),
                          nA + __popc(mm[2]) + __popc(mm[3] & lt)};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (vv[k]) scr_id[pos[k]] = static_cast<int16_t>(ev[k]);
      __syncwarp();
      // Compacted entry q (this lane's q = lane + 32 k): its id, whether it is
      // the id's first occurrence, and which rows list the id.
      int idq[4];
      unsigned mkq[4];
      bool fq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int q = lane + 32 * k;
        idq[k] = -1;
        mkq[k] = 0;
        fq[k] = false;
        if (q < nall) {
          const int id = scr_id[q];
          bool f = true;
          unsigned m = 0;
          for (int w = 0; w < nall; ++w)
            if (scr_id[w] == id) {
              if (w < q) f = false;
              m |= w < nA ? 1u : 2u;
            }
          idq[k] = id;
          mkq[k] = m;
          fq[k] = f;
          scr_first[q] = f ? 1 : 0;
        }
      }
      int nu = 0;
#pragma unroll
      for (int k = 0; k < 4; ++k) nu += __popc(__ballot_sync(0xffffffffu, fq[k]));
      if (lane == 0) {
        u_unit(slot) = t;
        u_hdr(slot, 0) = static_cast<int16_t>(nA);
        u_hdr(slot, 1) = static_cast<int16_t>(nB);
        u_hdr(slot, 2) = static_cast<int16_t>(nu);
        u_hdr(slot, 3) = -1;
      }
      __syncwarp();
      // A first occurrence's union position: the distinct ids below it.
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (!fq[k]) continue;
        int rank = 0;
        for (int w = 0; w < nall; ++w) rank += (scr_first[w] && scr_id[w] < idq[k]) ? 1 : 0;
        u_id(slot, rank) = static_cast<int16_t>(idq[k]);
        u_mask(slot, rank) = static_cast<uint8_t>(mkq[k]);
        if (idq[k] == j) u_hdr(slot, 3) = static_cast<int16_t>(rank);
      }
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bTFull + slot));
    }
    if (!ok && lane == 0) fail();
  } else if (warp == 0) {
    // ------------------------------------------------------------ Q, K loads
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      int itv = 0, E = 0;                      // non-empty units, union blocks whose K was loaded
      int last_q[2] = {-1, -1};                // last unit whose Q each buffer received
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const int t = u_unit(slot);
        if (t < 0) break;
        const int nA = u_hdr(slot, 0), nB = u_hdr(slot, 1), nu = u_hdr(slot, 2);
        int b, hkv, p, j;
        decode(t, b, hkv, p, j);
        const int hqA = hkv * g + 2 * p, tok0 = b * a.S;
        if (nu > 0) {
          const int qs = itv % C::kQBuf;
          if (itv >= C::kQBuf && !wait_bar(BAR(C::bQEmpty + qs), ((itv / C::kQBuf) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_expect_tx(BAR(C::bQFull + qs), ((nA > 0 ? 1 : 0) + (nB > 0 ? 1 : 0)) * C::kTile);
          for (int x = 0; x < 2; ++x) {
            if ((x == 0 ? nA : nB) == 0) continue;
#pragma unroll
            for (int gg = 0; gg < D / 64; ++gg)
              tma_load_3d(sQ + (qs * 2 + x) * C::kTile + gg * C::kRegion, &tmQ, BAR(C::bQFull + qs), gg * 64,
                          hqA + x, tok0 + j * BS);
          }
          last_q[qs] = itv;
          ++itv;
          for (int n = 0; n < nu && ok; ++n, ++E) {
            const int ks = E % C::kKSlots;
            if (E >= C::kKSlots && !wait_bar(BAR(C::bKEmpty + ks), ((E / C::kKSlots) - 1) & 1, abort_flag)) {
              ok = false;
              break;
            }
            const uint32_t bar = BAR(C::bKFull + ks);
            mbar_expect_tx(bar, C::kTile);
            const int id = u_id(slot, n);
#pragma unroll
            for (int gg = 0; gg < D / 64; ++gg)
              tma_load_3d(sK + gg * C::kKRing + ks * C::kRegion, &tmK, bar, gg * 64, hkv, tok0 + id * BS);
          }
        }
        if (ok) mbar_arrive(BAR(C::bTEmpty + slot));
      }
      if (!ok) {
        fail();
        for (int k = 0; k < C::kKSlots; ++k) {
          int last = -1;
          for (int n = k; n < E; n += C::kKSlots) last = n;
          if (last >= 0) mbar_wait(BAR(C::bKFull + k), (last / C::kKSlots) & 1, kWaitNs);
        }
        for (int k = 0; k < C::kQBuf; ++k)
          if (last_q[k] >= 0) mbar_wait(BAR(C::bQFull + k), (last_q[k] / C::kQBuf) & 1, kWaitNs);
      }
    }
  } else if (warp == 10) {
    // ------------------------------------------------------------ V loads
    if (lane == 0) {
      prefetch_tmap(&tmV);
      int E = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const int slot = it % kSlots;
        if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
        const int t = u_unit(slot);
        if (t < 0) break;
        int b, hkv, p, j;
        decode(t, b, hkv, p, j);
        const int nu = u_hdr(slot, 2), tok0 = b * a.S;
        for (int n = 0; n < nu && ok; ++n, ++E) {
          const int vs = E % C::kVSlots;
          if (E >= C::kVSlots && !wait_bar(BAR(C::bVEmpty + vs), ((E / C::kVSlots) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t bar = BAR(C::bVFull + vs);
          mbar_expect_tx(bar, C::kTile);
          const int id = u_id(slot, n);
#pragma unroll
          for (int gg = 0; gg < D / 64; ++gg)
            tma_load_3d(sV + vs * C::kTile + gg * C::kRegion, &tmV, bar, gg * 64, hkv, tok0 + id * BS);
        }
        if (ok) mbar_arrive(BAR(C::bTEmpty + slot));
      }
      if (!ok) {
        fail();
        for (int k = 0; k < C::kVSlots; ++k) {
          int last = -1;
          for (int n = k; n < E; n += C::kVSlots) last = n;
          if (last >= 0) mbar_wait(BAR(C::bVFull + k), (last / C::kVSlots) & 1, kWaitNs);
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BS, BS, 0, 0);     // 128 rows x 128 keys
      constexpr uint32_t idPV = idesc_bf16_f32(BS, D, 0, 1);     // P K-major in TMEM, V MN-major
      const uint64_t dQ0 = smem_desc_sw128(sQ, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sK, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sV, C::kRegion, 1024);
      Step q[2];                 // steps whose S is issued and PV is not; q[0] the older
      int qn = 0;
      int it = 0, slot = 0, nu = 0, e = 0, x = 0, seen = 0, qs = 0;
      bool have = false, more = true, first_unit = false;
      int vgS = 0, ES = 0, itvS = 0;   // S cursor: steps issued, union blocks done, non-empty units entered
      int EP = 0;                      // union blocks whose PV is done
      bool ok = true;
      while (ok) {
        // S runs one step ahead of PV, across unit boundaries.
        while (ok && more && qn < 2) {
          if (!have) {
            slot = it % kSlots;
            if (!wait_bar(BAR(C::bTFull + slot), (it / kSlots) & 1, abort_flag)) { ok = false; break; }
            if (u_unit(slot) < 0) { more = false; break; }
            nu = u_hdr(slot, 2);
            if (nu == 0) {                       // nothing to compute: release the descriptor now
              mbar_arrive(BAR(C::bTEmpty + slot));
              ++it;
              continue;
            }
            have = true;
            e = 0;
            x = (u_mask(slot, 0) & 1) ? 0 : 1;
            seen = 0;
            first_unit = true;
            qs = itvS % C::kQBuf;
            if (!wait_bar(BAR(C::bQFull + qs), (itvS / C::kQBuf) & 1, abort_flag)) { ok = false; break; }
          }
          const unsigned mk = u_mask(slot, e);
          Step st;
          st.slot = slot;
          st.x = x;
          st.vg = vgS;
          st.itv = itvS;
          st.first_entry = x == 0 || !(mk & 1u);
          st.last_entry = x == 1 || !(mk & 2u);
          st.first_unit = first_unit;
          st.first_x = !(seen & (1 << x));
          st.last_unit = st.last_entry && e == nu - 1;
          const int ks = ES % C::kKSlots;
          if (st.first_entry && !wait_bar(BAR(C::bKFull + ks), (ES / C::kKSlots) & 1, abort_flag)) { ok = false; break; }
          // The S buffer holds the P of step vgS - 2 until that step's PV completes.
          if (vgS >= 2 && !wait_bar(BAR(C::bPVDone + (vgS & 1)), ((vgS - 2) >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t tS = tmem + C::kColS + (vgS & 1) * 128;
          const uint64_t dq = dQ0 + ((qs * 2 + x) * C::kTile) / 16, dk = dK0 + ks * (C::kRegion / 16);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t qoff = ((kk / 4) * C::kRegion + (kk % 4) * 32) / 16;
            const uint32_t koff = (kk / 4) * (C::kKRing / 16) + (kk % 4) * 2;
            if (kk == 0) mma_bf16_c<false>(tS, dq + qoff, dk + koff, idS);
            else mma_bf16_c<true>(tS, dq + qoff, dk + koff, idS);
          }
          mma_commit(BAR(C::bSFull + (vgS & 1)));
          if (st.last_entry) {
            mma_commit(BAR(C::bKEmpty + ks));
            ++ES;
          }
          seen |= 1 << x;
          first_unit = false;
          ++vgS;
          q[qn++] = st;
          if (!st.last_entry) {
            x = 1;
          } else if (e + 1 < nu) {
            ++e;
            x = (u_mask(slot, e) & 1u) ? 0 : 1;
          } else {                               // every S of the unit issued: its Q buffer frees
            mma_commit(BAR(C::bQEmpty + qs));
            ++itvS;
            ++it;
            have = false;
          }
        }
        if (!ok || qn == 0) break;
        // PV of the older queued step.
        const Step st = q[0];
        const int vs = EP % C::kVSlots;
        if (!wait_bar(BAR(C::bPFull + (st.vg & 1)), (st.vg >> 1) & 1, abort_flag)) { ok = false; break; }
        if (st.first_unit && st.itv >= 1 && !wait_bar(BAR(C::bOFree), (st.itv - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (st.first_entry && !wait_bar(BAR(C::bVFull + vs), (EP / C::kVSlots) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t tO = tmem + C::kColO + st.x * D;
        const uint32_t tP = tmem + C::kColS + (st.vg & 1) * 128;
        const uint64_t dv = dV0 + vs * (C::kTile / 16);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk) {
          // Keys 16 kk ..: the P of keys 64 h .. 64 h + 63 sits in columns 64 h .. 64 h + 31.
          const uint32_t pa = tP + 64 * (kk / 4) + 8 * (kk % 4);
          if (kk == 0 && st.first_x) mma_bf16_ts<false>(tO, pa, dv + kk * 128, idPV);
          else mma_bf16_ts<true>(tO, pa, dv + kk * 128, idPV);
        }
        mma_commit(BAR(C::bPVDone + (st.vg & 1)));
        if (st.last_entry) {
          mma_commit(BAR(C::bVEmpty + vs));
          ++EP;
        }
        if (st.last_unit) {
          mma_commit(BAR(C::bOFull));
          mbar_arrive(BAR(C::bTEmpty + st.slot));
        }
        q[0] = q[1];
        --qn;
      }
      if (!ok) fail();
      // Everything this thread issued has completed once bFin fires.
      mma_commit(BAR(C::bFin));
      mbar_wait(BAR(C::bFin), 0, kWaitNs);
    }
  } else {
    // ------------------------------------------------------------- softmax
    const int sp = warp & 3;                          // TMEM subpartition
    const int half = (warp - 2) >> 2;                 // which 64 of a step's 128 key columns
    const int r = sp * 32 + lane;                     // query row in the block
    const uint32_t lane_base = static_cast<uint32_t>(sp * 32) << 16;
    // Waits give the same answer in every lane.
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
    // This warp's output columns: (D/2) half + 32 i, i < D/64.
    constexpr int kOParts = D / 64;
    auto o_col = [&](int i) { return (D / 2) * half + 32 * i; };
    auto zero_row = [&](__nv_bfloat16* out) {
#pragma unroll
      for (int i = 0; i < kOParts; ++i)
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) *reinterpret_cast<uint4*>(out + o_col(i) + q8 * 8) = make_uint4(0, 0, 0, 0);
    };
    bool pend = false;
    int pend_itv = 0;
    float pend_l0 = 0.f, pend_l1 = 0.f, pend_m0 = 0.f, pend_m1 = 0.f;
    bool pend_has0 = false, pend_has1 = false;
    __nv_bfloat16* pend_out = nullptr;                // the first head's row; the second's is + D
    float* pend_lse = nullptr;                        // the first head's normaliser; the second's is + S
    auto epilogue = [&]() -> bool {
      if (!wwait(C::bOFull, pend_itv & 1)) return false;
      xl[(0 * 2 + half) * BS + r] = pend_l0;
      xl[(1 * 2 + half) * BS + r] = pend_l1;
      if (!exchange()) return false;
      tc_fence_after();
      // Each row's D/2 output columns of this warp go through a 2 KB staging
      // area so that a global store covers whole 128-byte row segments (a
      // store straight from the registers would touch 32 rows at once).
      constexpr int kChunks = D / 16;                 // 16-byte chunks of a half row
      constexpr int kRowsPass = 2048 / (16 * kChunks);
      constexpr int kRowsIns = 32 / kChunks;          // rows per coalesced store
      uint8_t* stage = sm + C::kOffStage + (warp - 2) * 2048;
      const size_t row_stride = static_cast<size_t>(a.Hq) * D;
#pragma unroll 1
      for (int x = 0; x < 2; ++x) {
        if (!(x == 0 ? pend_has0 : pend_has1)) continue;
        const float l = (x == 0 ? pend_l0 : pend_l1) + xl[(x * 2 + 1 - half) * BS + r];
        const float inv = 1.f / l;
        if constexpr (kLse)
          if (half == 0)
            pend_lse[static_cast<size_t>(x) * a.S] = ((x == 0 ? pend_m0 : pend_m1) + __log2f(l)) * 0.6931471805599453f;
        const uint32_t tO = tmem + lane_base + C::kColO + x * D + (D / 2) * half;
        uint4 w[kChunks];
#pragma unroll
        for (int i = 0; i < kOParts; ++i) {
          float o[32];
          tmem_ld32(tO + 32 * i, o);
          tmem_ld_wait();
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8)
            w[i * 4 + q8] = make_uint4(pack_bf16(o[q8 * 8 + 0] * inv, o[q8 * 8 + 1] * inv),
                                       pack_bf16(o[q8 * 8 + 2] * inv, o[q8 * 8 + 3] * inv),
                                       pack_bf16(o[q8 * 8 + 4] * inv, o[q8 * 8 + 5] * inv),
                                       pack_bf16(o[q8 * 8 + 6] * inv, o[q8 * 8 + 7] * inv));
        }
        // Row 0 of this warp (lane 0's row), head x, this warp's first column.
        __nv_bfloat16* out0 = pend_out - static_cast<size_t>(lane) * row_stride + x * D + (D / 2) * half;
#pragma unroll
        for (int pass = 0; pass < 32 / kRowsPass; ++pass) {
          const int rl = lane - pass * kRowsPass;
          if (rl >= 0 && rl < kRowsPass) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
              *reinterpret_cast<uint4*>(stage + rl * 16 * kChunks + ((c ^ rl) % kChunks) * 16) = w[c];
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < kRowsPass / kRowsIns; ++i) {
            const int rr = i * kRowsIns + lane / kChunks, c = lane % kChunks;
            const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * 16 * kChunks + ((c ^ rr) % kChunks) * 16);
            *reinterpret_cast<uint4*>(out0 + static_cast<size_t>(pass * kRowsPass + rr) * row_stride + c * 8) = v;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bOFree));
      pend = false;
      return true;
    };
    int vg = 0, itv = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int slot = it % kSlots;
      if (!wwait(C::bTFull + slot, (it / kSlots) & 1)) { ok = false; break; }
      const int t = u_unit(slot);
      if (t < 0) break;
      const int nA = u_hdr(slot, 0), nB = u_hdr(slot, 1), nu = u_hdr(slot, 2), diag = u_hdr(slot, 3);
      int b, hkv, p, j;
      decode(t, b, hkv, p, j);
      const int hqA = hkv * g + 2 * p;
      const bool hasB = 2 * p + 1 < g;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                           ((static_cast<size_t>(b) * a.S + static_cast<size_t>(j) * BS + r) * a.Hq + hqA) * D;
      float* lse = kLse ? a.lse + (static_cast<size_t>(b) * a.Hq + hqA) * a.S + static_cast<size_t>(j) * BS + r
                        : nullptr;
      if (nA == 0) zero_row(out);                     // a head with nothing selected: zero output
      if (hasB && nB == 0) zero_row(out + D);
      if (kLse && half == 0) {
        if (nA == 0) lse[0] = -INFINITY;
        if (hasB && nB == 0) lse[a.S] = -INFINITY;
      }
      if (nu == 0) {
        __syncwarp();
        if (lane == 0) mbar_arrive(BAR(C::bTEmpty + slot));
        continue;
      }
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;   // running max (log2 units), sum per head
      bool first0 = true, first1 = true, unit_first = true;
      for (int e = 0; e < nu && ok; ++e) {
        const unsigned mk = u_mask(slot, e);
#pragma unroll 1
        for (int x = 0; x < 2; ++x) {
          if (!(mk & (1u << x))) continue;
          if (!wwait(C::bSFull + (vg & 1), (vg >> 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t tS = tmem + lane_base + C::kColS + (vg & 1) * 128;
          float sv[64];
          tmem_ld32(tS + 64 * half, sv);
          tmem_ld32(tS + 64 * half + 32, sv + 32);
          tmem_ld_wait();
          if (e == diag) {                            // the query's own block: keys after the row
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (64 * half + c > r) sv[c] = -INFINITY;
          }
          float pmax = -INFINITY;
#pragma unroll
          for (int c = 0; c < 64; ++c) pmax = fmaxf(pmax, sv[c]);
          float* xg = xch + (vg & 1) * 2 * BS;
          xg[half * BS + r] = pmax;
          if (!exchange()) { ok = false; break; }
          const float mb = fmaxf(pmax, xg[(1 - half) * BS + r]) * sl2;
          float m_used = x == 0 ? m0 : m1, l_sum = x == 0 ? l0 : l1;
          const bool first = x == 0 ? first0 : first1;
          float alpha = 1.f;
          bool rescale = false;
          if (mb > m_used + 8.f) {
            alpha = ex2_approx(m_used - mb);
            rescale = !first;
            m_used = mb;
            l_sum *= alpha;
          }
          // P of keys 64 half .. as bf16 pairs (computed first: S is dead after it).
          uint32_t pw[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2_approx(__fmaf_rn(sv[2 * c], sl2, -m_used));
            const float p1 = ex2_approx(__fmaf_rn(sv[2 * c + 1], sl2, -m_used));
            l_sum += p0 + p1;
            pw[c] = pack_bf16(p0, p1);
          }
          // O_x holds every PV before this step once the previous step's completes.
          const bool need_o = __any_sync(0xffffffffu, rescale);
          if (need_o) {
            if (!wwait(C::bPVDone + ((vg - 1) & 1), ((vg - 1) >> 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tO = tmem + lane_base + C::kColO + x * D + (D / 2) * half;
#pragma unroll
            for (int i = 0; i < kOParts; ++i) {
              float o[32];
              tmem_ld32(tO + 32 * i, o);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] *= alpha;
              tmem_st32(tO + 32 * i, o);
            }
          }
          // P into columns 64 half .. 64 half + 31 of the same S buffer (only
          // this warp read them).
          tmem_st32(tS + 64 * half, reinterpret_cast<const float*>(pw));
          tmem_st_wait();
          if (x == 0) { m0 = m_used; l0 = l_sum; first0 = false; }
          else { m1 = m_used; l1 = l_sum; first1 = false; }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(BAR(C::bPFull + (vg & 1)));
          ++vg;
          if (unit_first && pend && !epilogue()) { ok = false; break; }
          unit_first = false;
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(BAR(C::bTEmpty + slot));
      pend = true;
      pend_itv = itv;
      pend_l0 = l0;
      pend_l1 = l1;
      pend_m0 = m0;
      pend_m1 = m1;
      pend_lse = lse;
      pend_has0 = nA > 0;
      pend_has1 = hasB && nB > 0;
      pend_out = out;
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

template <int D>
cudaError_t launch_union(const AttendArgs& a, cudaStream_t st) {
  using C = UCfg<D>;
  CUtensorMap mq, mk, mv;
  const long long rows = static_cast<long long>(a.B) * a.S;
  if (!make_tile_map(&mq, a.q, rows, a.Hq, D, C::BS) || !make_tile_map(&mk, a.k, rows, a.Hkv, D, C::BS) ||
      !make_tile_map(&mv, a.v, rows, a.Hkv, D, C::BS))
    return cudaErrorInvalidValue;
  auto k = a.lse ? attend_union_kernel<D, true> : attend_union_kernel<D, false>;
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(k), C::kSmem);
  if (e != cudaSuccess) return e;
  const int sms = cached_sm_count();
  if (sms <= 0) return cudaErrorUnknown;
  const int g = a.Hq / a.Hkv;
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return cudaErrorInvalidValue;
  const long long nunits = static_cast<long long>(a.B) * a.Hkv * ((g + 1) / 2) * nbr;
  // 512 tensor-memory columns: one CTA per SM.
  const unsigned grid = static_cast<unsigned>(nunits < sms ? nunits : sms);
  // Every CTA takes one unit number past the last: the counter reaches nunits + grid.
  if (!a.tile_counter || nunits + grid > 0x7fffffffLL || a.nsel > 64) return cudaErrorInvalidValue;
  e = launch_pdl(k, dim3(grid), dim3(kThreads), C::kSmem, st, mq, mk, mv, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_union(const AttendArgs& a, cudaStream_t st) {
  if (a.bs != 128 || a.Hq % a.Hkv != 0) return cudaErrorInvalidValue;
  if (a.D == 64) return launch_union<64>(a, st);
  if (a.D == 128) return launch_union<128>(a, st);
  return cudaErrorInvalidValue;
}

}  // namespace mdr
