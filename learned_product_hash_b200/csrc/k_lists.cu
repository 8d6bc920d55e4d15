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
// This is a stable counting sort by (address, block id).  One warp walks the
// blocks 32 at a time in order; lanes with equal addresses find each other
// with __match_any_sync, the lowest of them adds the group's size to the
// address's shared-memory counter (a warp-aggregated atomic) and every lane's
// rank is that counter's old value plus its rank inside the group.  The other
// warps meanwhile pad the lists with -1.

#include "common.cuh"
#include "kernels.h"

namespace mdr {

__global__ void __launch_bounds__(1024)
lists_kernel(const ListsArgs a) {
  extern __shared__ int32_t cnt[];                 // [A]
  __shared__ int32_t s_ovf, s_max;
  const int bh = blockIdx.x;
  const size_t nlist = static_cast<size_t>(a.A) * a.cap;
  int32_t* lists = a.lists + static_cast<size_t>(bh) * nlist;
  const int32_t* addr = a.addr + static_cast<size_t>(bh) * a.nb;
  const int tid = threadIdx.x, lane = tid & 31;

  for (int x = tid; x < a.A; x += blockDim.x) cnt[x] = 0;
  if (tid == 0) { s_ovf = 0; s_max = 0; }
  if ((nlist & 3) == 0 && (reinterpret_cast<uintptr_t>(lists) & 15) == 0) {
    int4* l4 = reinterpret_cast<int4*>(lists);
    const int4 m1 = make_int4(-1, -1, -1, -1);
    for (size_t x = tid; x < nlist / 4; x += blockDim.x) l4[x] = m1;
  } else {
    for (size_t x = tid; x < nlist; x += blockDim.x) lists[x] = -1;
  }
  __syncthreads();

  if (tid < 32) {
    for (int base = 0; base < a.nb; base += 32) {
      const int i = base + lane;
      const bool valid = i < a.nb;
      const unsigned vm = __ballot_sync(0xffffffffu, valid);
      if (valid) {
        const int ad = addr[i];
        const unsigned peers = __match_any_sync(vm, ad);
        const int leader = __ffs(peers) - 1;
        const int inner = __popc(peers & ((1u << lane) - 1u));
        int before = 0;
        if (lane == leader) before = atomicAdd(&cnt[ad], __popc(peers));
        before = __shfl_sync(peers, before, leader);
        const int rank = before + inner;
        if (rank < a.cap) lists[static_cast<size_t>(ad) * a.cap + rank] = i;
      }
      __syncwarp();
    }
  }
  __syncthreads();

  int ovf = 0, mx = 0;
  int32_t* load = a.load + static_cast<size_t>(bh) * a.A;
  for (int x = tid; x < a.A; x += blockDim.x) {
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
  const size_t smem = static_cast<size_t>(a.A) * sizeof(int32_t);
  cudaError_t e = cudaFuncSetAttribute(lists_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  lists_kernel<<<a.B * a.H, 1024, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace mdr
