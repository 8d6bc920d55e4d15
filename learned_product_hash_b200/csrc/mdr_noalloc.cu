// mdr_route_noalloc: the route step for callers that cannot allocate.
//
// Some callers cannot hand the library a workspace and cannot call cudaMalloc
// either: a serving loop whose device memory is reserved up front by its own
// pool, or a plugin interface that passes an operator nothing but its input
// and output buffers.  cudaMalloc may also synchronise the device and take
// unbounded time, which such callers cannot afford mid-stream.  For them the
// route step (query summaries, probe codewords, rerank, top-R) runs with its
// scratch -- the query block means and the probed codewords -- in a fixed
// array compiled into this library.
//
// The array is a file-scope __device__ variable of kNoAllocScratchBytes
// (32 MiB): every GPU that loads the library holds it until the process
// exits.  Host code cannot use the array's name as a device address, so the
// first call on each device, with that device current, looks the address up
// with cudaGetSymbolAddress and caches it; make that first call before any
// stream capture.  All calls share the array: two calls whose work overlaps
// on the GPU (different streams, or different host threads) race on it.
// Nothing in it has to start at zero: the summary kernel writes every entry
// the route kernel later reads.

#include <cmath>
#include <cstring>
#include <mutex>

#include "mdr.h"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device address of the scratch array on the current device (looked up once
// per device).  Returns nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" mdr_status mdr_route_noalloc(const mdr_config* cfg, const void* q, const float* codebooks,
                                        const mdr_index* idx, int32_t* sel, int32_t* ncand, void* stream) {
  const mdr_status st = mdr_check_config(cfg);
  if (st != MDR_OK) return st;
  if (!q || !codebooks || !sel || (reinterpret_cast<uintptr_t>(q) & 15) != 0) return MDR_ERR_INVALID_ARG;
  if (!idx || !idx->kbar || !idx->lists || !idx->load) return MDR_ERR_INVALID_ARG;

  const size_t nb = static_cast<size_t>(cfg->S / cfg->block);
  const size_t routes = static_cast<size_t>(cfg->B) * cfg->Hq * nb;
  const size_t qbar_bytes = round256(routes * cfg->D * sizeof(float));
  const size_t codes_bytes = round256(routes * cfg->P * cfg->probes * sizeof(int32_t));
  if (qbar_bytes + codes_bytes > kNoAllocScratchBytes) return MDR_ERR_WORKSPACE;   // too large for the array

  uint8_t* scratch = static_cast<uint8_t*>(scratch_on_current_device());
  if (!scratch) return MDR_ERR_CUDA;
  float* qbar = reinterpret_cast<float*>(scratch);
  int32_t* qcodes = reinterpret_cast<int32_t*>(scratch + qbar_bytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  mdr::SummarizeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.x[0] = q;
  a.xbar[0] = qbar;
  a.qcodes = qcodes;
  a.H[0] = cfg->Hq;
  a.H[1] = cfg->Hkv;
  a.codebooks = codebooks;
  a.B = cfg->B; a.S = cfg->S; a.D = cfg->D; a.bs = cfg->block; a.nb = static_cast<int>(nb);
  a.P = cfg->P; a.K = cfg->K; a.probes = cfg->probes;
  for (int i = 0; i < cfg->D / 2; ++i)
    a.inv_freq[i] = static_cast<float>(std::pow(static_cast<double>(cfg->rope_base), -2.0 * i / cfg->D));
  if (mdr::launch_summarize(a, cfg->dtype == MDR_BF16, s) != cudaSuccess) return MDR_ERR_CUDA;

  int A = 1;
  for (int p = 0; p < cfg->P; ++p) A *= cfg->K;
  mdr::RouteArgs ra{};
  ra.qbar = qbar; ra.qcodes = qcodes; ra.kbar = idx->kbar; ra.lists = idx->lists; ra.load = idx->load;
  ra.sel = sel; ra.ncand = ncand;
  ra.B = cfg->B; ra.Hq = cfg->Hq; ra.Hkv = cfg->Hkv; ra.nb = static_cast<int>(nb); ra.D = cfg->D;
  ra.P = cfg->P; ra.K = cfg->K; ra.A = A; ra.probes = cfg->probes; ra.cap = cfg->cap;
  ra.R = cfg->R; ra.L = cfg->L;
  return mdr::launch_route(ra, s) == cudaSuccess ? MDR_OK : MDR_ERR_CUDA;
}
