// K1: rotary embedding and per-block summaries.
//
// For every token block j of sequence b and every head of each side (side 0:
// queries, Hq heads; side 1: keys, Hkv heads) the kernel rotates the block's
// bs tokens, optionally writes the rotated copy (the attention kernel reads
// it) and averages them into the block summary ("Monodratic: a reproducible
// sparse attention mixer", section Mixer: routing acts on rotated keys and
// queries, summarised per block).  The codes of the summaries are K2
// (k_codes.cu), launched right after by launch_summarize.
//
// Rotary convention: coordinate i pairs with i + D/2; the pair at absolute
// position t turns by the float32 angle fp32(t) * omega_i, with omega_i =
// base^(-2i/D) rounded to float32 on the host; cosine and sine by sincosf.
//
// Layout of the work.  The kernel is a persistent stream over units; a unit
// is (b, j, side, head group), a head group being up to 256 / (D / 2 / V)
// consecutive heads (V elements per 16 bytes), so that one thread owns one
// (head, 16-byte chunk) of both halves of a head row.  Each CTA takes a
// contiguous range of units, so that the query and key units of a block
// follow each other and share its rotation table.  Per unit the block's rows
// of those heads arrive in chunks of up to 32 KB through a ring of
// shared-memory stages, filled with bulk copies by one producer thread that
// runs ahead across units.  The 256 consumer threads (eight warps: with the
// producer warp at most three warps share a scheduler, which leaves room for
// 168 registers a thread and four tokens in flight per thread)
//   1. build the block's (cos, sin) table in shared memory, laid out so that
//      the eight lanes reading one token's chunk table hit distinct banks;
//   2. per chunk, rotate their (token, head, chunk) pieces, write them to the
//      rotated copy with 16-byte stores, and add them to float32 running
//      sums (token group tg takes tokens tg, tg + TG, ... in order);
//   3. sum the token groups in order 0, 1, ... TG-1 and scale by 1/bs into
//      the block mean (float32), written to the summaries.
// The read traffic is one pass over q and k, the write traffic the rotated
// copies plus the (small) summaries.
//
// Every wait is bounded (2 s of wall time) and gives up once another thread
// has given up; a wait that runs out writes status 1 (if a status word was
// given), and the producer waits (bounded) for its copies in flight.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace mdr {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;      // 256
constexpr int kSumThreads = kConsumers + 32;         // + the producer warp
constexpr int kMaxStages = 6;
constexpr int kMaxRowBytes = 16384;     // one token's row of a head group
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr int kSmemLimit = 232448;

// Host-computed plan of a launch.
struct SumPlan {
  int esize, V, CH, half, log2_half;
  int HG[2];          // heads per group
  int ng[2];          // head groups per side (0: side skipped)
  int NG;             // ng[0] + ng[1]
  int nunits;         // B * nb * NG
  int nst;            // ring stages
  int stage_bytes;    // 32 KB, or 16 KB when shared memory is short
  int off_tab, off_part, off_freq, off_ring, off_bar, smem;
};

__device__ __forceinline__ int pow2_floor(int x) { return 1 << (31 - __clz(x)); }

}  // namespace

template <typename T>
__global__ void __launch_bounds__(kSumThreads, 1)
summarize_kernel(const __grid_constant__ SummarizeArgs a, const SumPlan pl) {
  using E = Elem<T>;
  using namespace tc;
  constexpr int V = E::kVec;
  constexpr int esize = static_cast<int>(sizeof(T));
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int D = a.D, half = D / 2, CH = half / V, bs = a.bs;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full0 = sbase + pl.off_bar, empty0 = full0 + 8 * kMaxStages, cbar = empty0 + 8 * kMaxStages;
  int& abort_s = *reinterpret_cast<int*>(smem + pl.off_bar + 8 * (2 * kMaxStages + 1));
  volatile int* abort_flag = &abort_s;
  const int nst = pl.nst;

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, kConsumerWarps);
    }
    mbar_init(cbar, kConsumerWarps);
    fence_mbar_init();
    abort_s = 0;
  }
  __syncthreads();
  grid_dependency_wait();

  auto fail = [&]() {
    if (a.status) atomicExch(a.status, kDevWaitTimeout);
    *abort_flag = 1;
  };

  // Unit u: (b, j) = u / NG, group sg = u % NG (query groups first).
  struct Unit {
    int b, j, side, h0, HGa, rowbytes, TPC, nch;
  };
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;        // blocks a.j0 .. a.j0 + nbr - 1
  auto unit_of = [&](int u) {
    Unit x;
    const int bj = u / pl.NG;
    const int sg = u - bj * pl.NG;
    x.b = bj / nbr;
    x.j = a.j0 + (bj - x.b * nbr);
    x.side = sg < pl.ng[0] ? 0 : 1;
    const int hg = x.side ? sg - pl.ng[0] : sg;
    const int H = a.H[x.side];
    x.h0 = hg * pl.HG[x.side];
    x.HGa = min(pl.HG[x.side], H - x.h0);
    x.rowbytes = x.HGa * D * esize;
    x.TPC = min(bs, pow2_floor(pl.stage_bytes / x.rowbytes));
    x.nch = bs / x.TPC;
    return x;
  };

  // This CTA's units: a contiguous range, so that the query and key units of
  // a block follow each other and share the block's rotation table.
  const int u_begin = static_cast<int>(static_cast<long long>(blockIdx.x) * pl.nunits / gridDim.x);
  const int u_end = static_cast<int>(static_cast<long long>(blockIdx.x + 1) * pl.nunits / gridDim.x);

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;         // chunks issued
      int st = 0;             // stage of the next chunk
      uint32_t ph = 0;        // parity of the ring round it belongs to
      bool ok = true;
      for (int u = u_begin; u < u_end && ok; ++u) {
        const Unit x = unit_of(u);
        const int H = a.H[x.side];
        const T* src = static_cast<const T*>(a.x[x.side]);
        for (int ci = 0; ci < x.nch; ++ci) {
          // A stage is refilled once the consumers released it in the last round.
          if (issued >= nst && !mbar_wait_or_abort(empty0 + 8 * st, ph ^ 1u, abort_flag, kWaitNs)) {
            ok = false;
            break;
          }
          const uint32_t bar = full0 + 8 * st, dst = sbase + pl.off_ring + st * pl.stage_bytes;
          mbar_expect_tx(bar, static_cast<uint32_t>(x.TPC * x.rowbytes));
          const size_t tok0 = static_cast<size_t>(x.b) * a.S + static_cast<size_t>(x.j) * bs + ci * x.TPC;
          if (x.HGa == H) {           // the chunk's rows are contiguous
            bulk_load(dst, src + tok0 * H * D, static_cast<uint32_t>(x.TPC * x.rowbytes), bar);
          } else {
            for (int t = 0; t < x.TPC; ++t)
              bulk_load(dst + t * x.rowbytes, src + ((tok0 + t) * H + x.h0) * D, static_cast<uint32_t>(x.rowbytes),
                        bar);
          }
          ++issued;
          if (++st == nst) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        fail();
        for (int s = 0; s < nst; ++s) {   // the last copy issued into each stage
          int last = -1;
          for (int n = issued - 1; n >= 0 && n >= issued - nst; --n)
            if (n % nst == s) last = n;
          if (last >= 0) mbar_wait(full0 + 8 * s, static_cast<uint32_t>(last / nst) & 1u, kWaitNs);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  float4* tab4 = reinterpret_cast<float4*>(smem + pl.off_tab);   // [bs][V/2][CH]
  float4* part0 = reinterpret_cast<float4*>(smem + pl.off_part); // 2 x [TG][2V/4][combos]
  float* freq = reinterpret_cast<float*>(smem + pl.off_freq);    // omega_i
  int cph = 0;                 // consumer barrier phases completed
  auto cwait = [&](uint32_t bar, uint32_t par) {
    return __all_sync(0xffffffffu, mbar_wait_or_abort(bar, par, abort_flag, kWaitNs));
  };
  auto csync = [&]() -> bool {  // all consumer warps
    __syncwarp();
    if (lane == 0) mbar_arrive(cbar);
    const bool r = cwait(cbar, cph & 1);
    ++cph;
    return r;
  };
  const float inv_bs = 1.0f / static_cast<float>(bs);   // bs is a power of two
  int st = 0;                  // stage of the next chunk
  uint32_t ph = 0;             // parity of its ring round
  bool ok = true;
  for (int i = tid; i < half; i += kConsumers) freq[i] = a.inv_freq[i];
  int tab_j = -1;              // block whose table is in shared memory
  for (int u = u_begin; u < u_end && ok; ++u) {
    const Unit x = unit_of(u);
    const int H = a.H[x.side];
    // The key side's first head group pads this block's share of the
    // posting lists with -1 (the list kernel, which runs next, only scatters).
    if (x.side == 1 && x.h0 == 0 && a.lists_fill) {
      const size_t share = (a.lists_per_seq + a.nb - 1) / a.nb;
      const size_t lo = static_cast<size_t>(x.j) * share;
      const size_t hi = lo + share < a.lists_per_seq ? lo + share : a.lists_per_seq;
      int32_t* l = a.lists_fill + static_cast<size_t>(x.b) * a.lists_per_seq;
      for (size_t e = lo + tid; e < hi; e += kConsumers) l[e] = -1;
    }
    // 1. (cos, sin) of pair i at token t of the block: float4 (t, v2, c)
    //    holds pairs c*V + 2*v2 and c*V + 2*v2 + 1.  Rebuilt only when the
    //    block changes; every reader of the old table passed the barrier
    //    after the previous unit's chunks.
    if (x.j != tab_j) {
      if (tab_j < 0 && !csync()) { ok = false; break; }   // omega visible to all
#pragma unroll 4
      for (int e = tid; e < bs * half; e += kConsumers) {
        const int t = e >> pl.log2_half, i = e & (half - 1);
        const float ang = __fmul_rn(static_cast<float>(x.j * bs + t), freq[i]);
        float sn, cs;
        sincosf(ang, &sn, &cs);
        const int c = i / V, v = i % V;
        float* dst = reinterpret_cast<float*>(tab4 + (t * (V / 2) + v / 2) * CH + c) + 2 * (v & 1);
        dst[0] = cs;
        dst[1] = sn;
      }
      tab_j = x.j;
      if (!csync()) { ok = false; break; }
    }

    // 2. rotate, store, accumulate.
    const int combos = x.HGa * CH, TG = kConsumers / combos;
    const int combo = tid % combos, tg = tid / combos;
    const int hl = combo / CH, c = combo % CH;
    const bool active = tg < TG;
    T* __restrict__ xo = static_cast<T*>(a.xrot[x.side]);
    float s1[V], s2[V];
#pragma unroll
    for (int v = 0; v < V; ++v) { s1[v] = 0.f; s2[v] = 0.f; }
    for (int ci = 0; ci < x.nch; ++ci) {
      if (!cwait(full0 + 8 * st, ph)) { ok = false; break; }
      const uint8_t* stage = smem + pl.off_ring + st * pl.stage_bytes;
      if (active) {
#pragma unroll 4
        for (int tl = tg; tl < x.TPC; tl += TG) {
          const int t = ci * x.TPC + tl;
          const uint8_t* row = stage + tl * x.rowbytes + hl * D * esize;
          const uint4 r1 = *reinterpret_cast<const uint4*>(row + c * 16);
          const uint4 r2 = *reinterpret_cast<const uint4*>(row + half * esize + c * 16);
          float x1[V], x2[V], y1[V], y2[V];
          E::unpack(r1, x1);
          E::unpack(r2, x2);
          const float4* tr = tab4 + t * (V / 2) * CH + c;
#pragma unroll
          for (int v2 = 0; v2 < V / 2; ++v2) {
            const float4 cs = tr[v2 * CH];          // (cos, sin) of two pairs
            const int v = 2 * v2;
            y1[v] = __fmaf_rn(x1[v], cs.x, -__fmul_rn(x2[v], cs.y));
            y2[v] = __fmaf_rn(x2[v], cs.x, __fmul_rn(x1[v], cs.y));
            y1[v + 1] = __fmaf_rn(x1[v + 1], cs.z, -__fmul_rn(x2[v + 1], cs.w));
            y2[v + 1] = __fmaf_rn(x2[v + 1], cs.z, __fmul_rn(x1[v + 1], cs.w));
          }
#pragma unroll
          for (int v = 0; v < V; ++v) {
            s1[v] = __fadd_rn(s1[v], y1[v]);
            s2[v] = __fadd_rn(s2[v], y2[v]);
          }
          if (xo) {
            T* o = xo + ((static_cast<size_t>(x.b) * a.S + static_cast<size_t>(x.j) * bs + t) * H + x.h0 + hl) * D +
                   c * V;
            E::store(o, y1);
            E::store(o + half, y2);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
      if (++st == nst) { st = 0; ph ^= 1u; }
    }
    if (!ok) break;
    // Partial sums of this thread's token group into buffer u & 1: float4 e4
    // of its chunk pair (e4 < V/4: first half, otherwise second half).  That
    // buffer was last read two units ago, before the barrier that follows
    // the previous unit's partial sums.
    constexpr int NE4 = 2 * V / 4;
    float4* part4 = part0 + (u & 1) * (kConsumers * NE4);
    if (active) {
#pragma unroll
      for (int e4 = 0; e4 < NE4; ++e4) {
        const float* sp = e4 < V / 4 ? s1 + 4 * e4 : s2 + 4 * (e4 - V / 4);
        part4[(tg * NE4 + e4) * combos + combo] = make_float4(sp[0], sp[1], sp[2], sp[3]);
      }
    }
    if (!csync()) { ok = false; break; }

    // 3. block means.
    float* xbar = a.xbar[x.side];
    if (xbar) {
      for (int i = tid; i < combos * NE4; i += kConsumers) {
        const int e4 = i / combos, cb = i % combos;
        float4 sm = part4[e4 * combos + cb];
        for (int g = 1; g < TG; ++g) {
          const float4 p = part4[(g * NE4 + e4) * combos + cb];
          sm.x = __fadd_rn(sm.x, p.x); sm.y = __fadd_rn(sm.y, p.y);
          sm.z = __fadd_rn(sm.z, p.z); sm.w = __fadd_rn(sm.w, p.w);
        }
        sm.x *= inv_bs; sm.y *= inv_bs; sm.z *= inv_bs; sm.w *= inv_bs;
        const int h = cb / CH, cc = cb % CH;
        const int elem = e4 < V / 4 ? cc * V + 4 * e4 : half + cc * V + 4 * (e4 - V / 4);
        *reinterpret_cast<float4*>(xbar + ((static_cast<size_t>(x.b) * H + x.h0 + h) * a.nb + x.j) * D + elem) = sm;
      }
    }
  }
  if (!ok) fail();
}

namespace {

bool make_plan(const SummarizeArgs& a, bool bf16, SumPlan& pl) {
  pl.esize = bf16 ? 2 : 4;
  pl.V = 16 / pl.esize;
  pl.half = a.D / 2;
  pl.log2_half = 0;
  while ((1 << pl.log2_half) < pl.half) ++pl.log2_half;
  if ((1 << pl.log2_half) != pl.half) return false;
  pl.CH = pl.half / pl.V;
  if (pl.CH < 1 || pl.half % pl.V != 0) return false;
  const int max_heads = kConsumers / pl.CH;
  for (int s = 0; s < 2; ++s) {
    if (!a.x[s]) { pl.HG[s] = 1; pl.ng[s] = 0; continue; }
    pl.HG[s] = a.H[s] < max_heads ? a.H[s] : max_heads;
    pl.ng[s] = (a.H[s] + pl.HG[s] - 1) / pl.HG[s];
    const int rowbytes = pl.HG[s] * a.D * pl.esize;
    if (rowbytes > kMaxRowBytes || rowbytes % 16 != 0) return false;
  }
  pl.NG = pl.ng[0] + pl.ng[1];
  const int nbr = a.nbr > 0 ? a.nbr : a.nb;
  if (a.j0 < 0 || a.j0 + nbr > a.nb || (a.nbr <= 0 && a.j0 != 0)) return false;
  const long long nunits = static_cast<long long>(a.B) * nbr * pl.NG;
  if (nunits > 0x7fffffffLL) return false;
  pl.nunits = static_cast<int>(nunits);
  auto up = [](size_t x) { return (x + 127) / 128 * 128; };
  // Partial sums: two buffers of TG * combos <= 256 threads, 2V floats each.
  const size_t part = static_cast<size_t>(kConsumers) * 2 * pl.V * sizeof(float);
  pl.off_tab = 0;
  pl.off_part = static_cast<int>(up(static_cast<size_t>(a.bs) * pl.half * 2 * sizeof(float)));
  pl.off_freq = pl.off_part + static_cast<int>(2 * up(part));
  pl.off_ring = pl.off_freq + static_cast<int>(up(pl.half * sizeof(float)));
  const int bar_bytes = 8 * (2 * kMaxStages + 1) + 16;
  const int room = kSmemLimit - pl.off_ring - bar_bytes;
  pl.stage_bytes = room >= 4 * 32768 ? 32768 : 16384;
  pl.nst = std::min(kMaxStages, room / pl.stage_bytes);
  if (pl.nst < 2) return false;
  pl.off_bar = pl.off_ring + pl.nst * pl.stage_bytes;
  pl.smem = pl.off_bar + bar_bytes;
  return true;
}

}  // namespace

size_t summarize_smem_bytes(int bs, int D, int Hq, int Hkv) {
  SummarizeArgs a{};
  a.bs = bs; a.D = D; a.H[0] = Hq; a.H[1] = Hkv; a.B = 1; a.nb = 1;
  int dummy = 0;
  a.x[0] = &dummy; a.x[1] = &dummy;
  SumPlan pl{};
  return make_plan(a, true, pl) ? static_cast<size_t>(pl.smem) : 0;
}

cudaError_t launch_summarize(const SummarizeArgs& a, bool bf16, cudaStream_t st) {
  SumPlan pl{};
  if (!make_plan(a, bf16, pl)) return cudaErrorInvalidValue;
  if (pl.nunits == 0) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  const int sms = cached_sm_count();
  if (sms <= 0) return cudaErrorUnknown;
  const int grid = pl.nunits < sms ? pl.nunits : sms;
  if (bf16) {
    auto k = summarize_kernel<__nv_bfloat16>;
    if ((e = cached_allow_smem(reinterpret_cast<const void*>(k), pl.smem)) != cudaSuccess) return e;
    if ((e = launch_pdl(k, dim3(grid), dim3(kSumThreads), pl.smem, st, a, pl)) != cudaSuccess) return e;
  } else {
    auto k = summarize_kernel<float>;
    if ((e = cached_allow_smem(reinterpret_cast<const void*>(k), pl.smem)) != cudaSuccess) return e;
    if ((e = launch_pdl(k, dim3(grid), dim3(kSumThreads), pl.smem, st, a, pl)) != cudaSuccess) return e;
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // K2 on the summaries just written.
  CodesArgs c{};
  c.xbar[0] = a.qcodes ? a.xbar[0] : nullptr;
  c.xbar[1] = a.addr ? a.xbar[1] : nullptr;
  if (!c.xbar[0] && !c.xbar[1]) return cudaSuccess;
  c.H[0] = a.H[0]; c.H[1] = a.H[1];
  c.qcodes = a.qcodes; c.addr = a.addr; c.codebooks = a.codebooks;
  c.B = a.B; c.nb = a.nb; c.D = a.D; c.P = a.P; c.K = a.K; c.probes = a.probes;
  c.j0 = a.j0; c.nbr = a.nbr;
  return launch_codes(c, st);
}

}  // namespace mdr
