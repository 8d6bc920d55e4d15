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
// exits.  A second file-scope __device__ word holds the call's device status.
// Host code cannot use either name as a device address, so the first call on
// each device, with that device current, looks both addresses up with
// cudaGetSymbolAddress and caches them; that first call must not be made
// while its stream is capturing (it returns MDR_ERR_INVALID_ARG then).  All
// calls share the array and the word: two calls whose work overlaps on the
// GPU (different streams, or different host threads) race on them.  The
// status word is cleared at the start of every call (cudaMemsetAsync, which
// allocates nothing); nothing in the array has to start at zero, since the
// summary kernel writes every entry the route kernel later reads.
//
// If a bounded wait of the summary kernel runs out, that kernel sets the
// status word and the route kernel then writes -1 into every sel row and
// ncand entry instead of routing.  A normal route never does that (the last
// entry of a row is the query block itself), so sel[..., R+L-1] == -1 tells
// the caller the call failed on the device.

#include <cstring>
#include <mutex>

#include "mdr.h"
#include "kernels.h"
#include "abi_common.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) uint8_t g_route_scratch[kNoAllocScratchBytes];
__device__ __align__(16) int32_t g_route_status[4];

struct DeviceAddrs {
  void* scratch;
  int32_t* status;
};
DeviceAddrs g_addr[kMaxDevices] = {};
std::mutex g_addr_mu;

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Device addresses of the scratch array and the status word on the current
// device, looked up once per device.  The lookup is refused (invalid
// argument) while the stream is capturing; a failed lookup returns MDR_ERR_CUDA.
mdr_status addrs_on_current_device(cudaStream_t s, DeviceAddrs* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MDR_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (!g_addr[dev].scratch) {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return MDR_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return MDR_ERR_INVALID_ARG;   // first call during capture
    DeviceAddrs d{};
    if (cudaGetSymbolAddress(&d.scratch, g_route_scratch) != cudaSuccess) return MDR_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&d.status), g_route_status) != cudaSuccess)
      return MDR_ERR_CUDA;
    g_addr[dev] = d;
  }
  *out = g_addr[dev];
  return MDR_OK;
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

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceAddrs d{};
  const mdr_status ast = addrs_on_current_device(s, &d);
  if (ast != MDR_OK) return ast;
  uint8_t* scratch = static_cast<uint8_t*>(d.scratch);
  float* qbar = reinterpret_cast<float*>(scratch);
  int32_t* qcodes = reinterpret_cast<int32_t*>(scratch + qbar_bytes);
  if (cudaMemsetAsync(d.status, 0, sizeof(int32_t), s) != cudaSuccess) return MDR_ERR_CUDA;

  mdr::SummarizeArgs a;
  mdr::detail::fill_summarize_common(a, cfg, codebooks);
  a.x[0] = q;
  a.xbar[0] = qbar;
  a.qcodes = qcodes;
  a.status = d.status;
  if (mdr::launch_summarize(a, cfg->dtype == MDR_BF16, s) != cudaSuccess) return MDR_ERR_CUDA;

  mdr::RouteArgs ra = mdr::detail::route_args(cfg, qbar, qcodes, idx, sel, ncand);
  ra.upstream_status = d.status;
  return mdr::launch_route(ra, s) == cudaSuccess ? MDR_OK : MDR_ERR_CUDA;
}
