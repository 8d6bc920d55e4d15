// Host-side facts that every launch needs, looked up once per device: the
// SM count, the dynamic shared memory a kernel has been allowed, and a
// kernel's occupancy at a given block size and shared memory.  These runtime
// queries cost microseconds each; a forward makes a dozen of them, which
// would otherwise add to the host time of every call.

#include <mutex>
#include <vector>

#include "kernels.h"

namespace mdr {

namespace {

struct SmemEntry {
  int dev;
  const void* fn;
  int bytes;
};
struct OccEntry {
  int dev;
  const void* fn;
  int threads;
  size_t smem;
  int blocks;
};

std::mutex g_mu;
std::vector<int> g_sms;              // by device, 0 = not looked up
std::vector<SmemEntry> g_smem;
std::vector<OccEntry> g_occ;

}  // namespace

int cached_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (static_cast<int>(g_sms.size()) <= dev) g_sms.resize(dev + 1, 0);
  if (g_sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

cudaError_t cached_allow_smem(const void* fn, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const SmemEntry& s : g_smem)
    if (s.dev == dev && s.fn == fn && s.bytes >= bytes) return cudaSuccess;
  if ((e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes)) != cudaSuccess) return e;
  for (SmemEntry& s : g_smem)
    if (s.dev == dev && s.fn == fn) { s.bytes = bytes; return cudaSuccess; }
  g_smem.push_back({dev, fn, bytes});
  return cudaSuccess;
}

int cached_occupancy(const void* fn, int threads, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const OccEntry& o : g_occ)
    if (o.dev == dev && o.fn == fn && o.threads == threads && o.smem == smem) return o.blocks;
  int blocks = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, fn, threads, smem) != cudaSuccess) return 0;
  g_occ.push_back({dev, fn, threads, smem, blocks});
  return blocks;
}

}  // namespace mdr
