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
// This is a stable counting sort by (address, block id) in shared memory:
// all threads zero the per-address counts and stage the head's addresses;
// then one warp walks the blocks in order, 32 at a time: lanes with equal
// addresses find each other with __match_any_sync, a block's rank is the
// address's count so far plus the number of its peers in lower lanes, and the
// lowest peer adds the group's size to the count.  The walk is sequential in
// steps of 32, not in blocks, and needs no block-wide barrier.  The lists
// arrive padded with -1: the summary kernel of the key side, which runs just
// before on the same stream, writes the padding.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

constexpr int kListThreads = 256;

__global__ void __launch_bounds__(kListThreads)
lists_kernel(const ListsArgs a) {
  extern __shared__ int32_t cnt[];                 // [A] running counts, then [nb] addresses
  __shared__ int32_t s_ovf, s_max;
  grid_dependency_wait();
  const int bh = blockIdx.x;
  int32_t* lists = a.lists + static_cast<size_t>(bh) * static_cast<size_t>(a.A) * a.cap;
  const int j0 = a.j0, j1 = a.j1 > 0 ? a.j1 : a.nb, n = j1 - j0;   // blocks added
  const int32_t* addr = a.addr + static_cast<size_t>(bh) * a.nb + j0;
  const int tid = threadIdx.x, lane = tid & 31;
  int32_t* saddr = cnt + a.A;
  int32_t* load = a.load + static_cast<size_t>(bh) * a.A;

  // Counts so far: none, or the lists of blocks < j0.
  for (int x = tid; x < a.A; x += kListThreads) cnt[x] = j0 == 0 ? 0 : load[x];
  for (int x = tid; x < n; x += kListThreads) saddr[x] = addr[x];      // one coalesced read
  if (tid == 0) { s_ovf = 0; s_max = 0; }
  __syncthreads();

  if (tid < 32) {
    const unsigned lower = (1u << lane) - 1u;
    int ad_next = lane < n ? saddr[lane] : -1;
    for (int c0 = 0; c0 < n; c0 += 32) {
      const int i = c0 + lane;
      const int ad = ad_next;
      ad_next = i + 32 < n ? saddr[i + 32] : -1;
      const bool valid = i < n;
      const unsigned vm = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const unsigned peers = __match_any_sync(vm, ad);
        const int base = cnt[ad];
        const int rank = base + __popc(peers & lower);
        if (rank < a.cap) lists[static_cast<size_t>(ad) * a.cap + rank] = j0 + i;
        __syncwarp(vm);                            // every peer read the old count
        if ((peers & lower) == 0) cnt[ad] = base + __popc(peers);
      }
      __syncwarp();
    }
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
  if (a.j0 < 0 || a.j0 >= j1 || j1 > a.nb) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(a.A + (j1 - a.j0)) * sizeof(int32_t);
  cudaError_t e = cached_allow_smem(reinterpret_cast<const void*>(lists_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = launch_pdl(lists_kernel, dim3(a.B * a.H), dim3(kListThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace mdr
