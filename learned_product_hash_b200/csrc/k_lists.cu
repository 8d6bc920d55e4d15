// K3: bounded causal posting lists.
//
// One CTA per (sequence b, KV head h).  The blocks of the head are inserted
// in ascending block order: block i lands at position rank(i) of the list of
// its address, rank(i) = #{i' < i : addr[i'] == addr[i]}, and is stored when
// rank(i) < cap; otherwise it is an overflow event ("Monodratic: a
// reproducible sparse attention mixer", section Mixer: capacity-bounded,
// causal lists; section Capacity: overflow events and maximum assigned
// load).  Keeping the first cap blocks makes storage causal: whether block i
// is stored depends only on blocks before it.
//
// This is a stable counting sort by (address, block id) in shared memory,
// in rounds of 32 blocks per warp: (1) each warp takes 32 consecutive blocks,
// lanes with equal addresses find each other with __match_any_sync, a
// block's rank within its warp is the number of its peers in lower lanes,
// and the lowest peer records the group's size in the warp's row of a
// [warps][A] count table; (2) per address, a prefix over the warps turns the
// table into each warp's starting rank (the count so far plus the earlier
// warps' groups) and advances the running count; (3) each block lands at
// starting rank + rank within its warp.  The lists arrive padded with -1:
// the summary kernel of the key side, which runs just before on the same
// stream, writes the padding (or the caller clears them).

#include "common.cuh"
#include "kernels.h"

namespace mdr {

constexpr int kListThreads = 512;
constexpr int kListWarps = kListThreads / 32;

__global__ void __launch_bounds__(kListThreads)
lists_kernel(const ListsArgs a, const int nw) {
  extern __shared__ int32_t cnt[];                 // [A] running counts, then [nw][A] warp table
  __shared__ int32_t s_ovf, s_max;
  grid_dependency_wait();
  const int bh = blockIdx.x;
  int32_t* lists = a.lists + static_cast<size_t>(bh) * static_cast<size_t>(a.A) * a.cap;
  const int j0 = a.j0, j1 = a.j1 > 0 ? a.j1 : a.nb, n = j1 - j0;   // blocks added
  const int32_t* addr = a.addr + static_cast<size_t>(bh) * a.nb + j0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* cw = cnt + a.A;
  int32_t* load = a.load + static_cast<size_t>(bh) * a.A;
  const unsigned lower = (1u << lane) - 1u;

  // Counts so far: none, or the lists of blocks < j0.
  for (int x = tid; x < a.A; x += kListThreads) cnt[x] = j0 == 0 ? 0 : load[x];
  if (tid == 0) { s_ovf = 0; s_max = 0; }
  for (int r0 = 0; r0 < n; r0 += nw * 32) {
    for (int x = tid; x < nw * a.A; x += kListThreads) cw[x] = 0;
    __syncthreads();
    // (1) ranks within the warp's 32 blocks
    const int i = r0 + warp * 32 + lane;
    const bool valid = warp < nw && i < n;
    const int ad = valid ? addr[i] : -1;
    int rk = 0;
    if (warp < nw) {
      const unsigned vm = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const unsigned peers = __match_any_sync(vm, ad);
        rk = __popc(peers & lower);
        if (rk == 0) cw[warp * a.A + ad] = __popc(peers);
      }
    }
    __syncthreads();
    // (2) per address: each warp's starting rank, and the new running count
    for (int x = tid; x < a.A; x += kListThreads) {
      int run = cnt[x];
      for (int w = 0; w < nw; ++w) {
        const int t = cw[w * a.A + x];
        cw[w * a.A + x] = run;
        run += t;
      }
      cnt[x] = run;
    }
    __syncthreads();
    // (3) store the blocks that fit
    if (valid) {
      const int rank = cw[warp * a.A + ad] + rk;
      if (rank < a.cap) lists[static_cast<size_t>(ad) * a.cap + rank] = j0 + i;
    }
    __syncthreads();                               // the table is cleared for the next round
  }
  __syncthreads();

  int ovf = 0, mx = 0;
  for (int x = tid; x < a.A; x += kListThreads) {
    const int c = cnt[x];
    load[x] = c;
    ovf += c > a.cap ? c - a.cap : 0;
    mx = c > mx ? c : mx;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ovf += __shfl_xor_sync(0xffffffffu, ovf, o);
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) { atomicAdd(&s_ovf, ovf); atomicMax(&s_max, mx); }
  __syncthreads();
  if (tid == 0) { a.overflow[bh] = s_ovf; a.maxload[bh] = s_max; }
}

cudaError_t launch_lists(const ListsArgs& a, cudaStream_t st) {
  const int j1 = a.j1 > 0 ? a.j1 : a.nb;
  if (a.j0 < 0 || a.j0 >= j1 || j1 > a.nb || a.A < 1) return cudaErrorInvalidValue;
  // As many warp rows of the count table as fit next to the counts (A <= 16384: at least 2).
  constexpr int kSmemInts = 227 * 1024 / 4 - 64;
  int nw = (kSmemInts - a.A) / a.A;
  nw = nw < kListWarps ? nw : kListWarps;
  if (nw < 1) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(a.A) * (1 + nw) * sizeof(int32_t);
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(lists_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(lists_kernel, dim3(a.B * a.H), dim3(kListThreads), smem, st, a, nw);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
