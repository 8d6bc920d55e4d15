// C ABI of libmdr: argument checks, workspace carving and kernel launches.
// Declarations and the contract of every entry point are in include/mdr.h.

#include <cmath>
#include <cstring>
#include <mutex>

#include "mdr.h"
#include "kernels.h"
#include "abi_common.h"

namespace {

using mdr::SummarizeArgs;
using mdr::detail::ipow;

constexpr size_t kAlign = 256;
constexpr size_t kMaxDynamicSmem = 227 * 1024;    // per CTA on sm_100a

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
// The forward workspace starts with four int32 words, zeroed by every call
// before its first kernel: [0] the status word, [2] the attention kernel's
// tile counter.
constexpr size_t kStatusBytes = 4 * sizeof(int32_t);

size_t esize(const mdr_config* c) { return c->dtype == MDR_BF16 ? 2 : 4; }

bool is_pow2_in(int x, std::initializer_list<int> allowed) {
  for (int a : allowed)
    if (x == a) return true;
  return false;
}

mdr_status check(const mdr_config* c) {
  if (!c) return MDR_ERR_INVALID_ARG;
  if (c->B < 1 || c->S < 1 || c->Hq < 1 || c->Hkv < 1 || c->D < 1 || c->block < 1 || c->P < 1 ||
      c->K < 1 || c->cap < 1 || c->probes < 1 || c->R < 0 || c->L < 1)
    return MDR_ERR_INVALID_ARG;
  if (c->S % c->block != 0 || c->Hq % c->Hkv != 0 || c->D % c->P != 0 || c->probes > c->K)
    return MDR_ERR_INVALID_ARG;
  if (!(c->rope_base > 1.0f) || !(c->scale >= 0.0f) || !std::isfinite(c->rope_base) ||
      !std::isfinite(c->scale))
    return MDR_ERR_INVALID_ARG;
  if (c->dtype != MDR_F32 && c->dtype != MDR_BF16) return MDR_ERR_INVALID_ARG;
  if (!is_pow2_in(c->D, {32, 64, 128}) || !is_pow2_in(c->block, {16, 32, 64, 128}))
    return MDR_ERR_UNSUPPORTED;
  if (c->P > 4 || (c->D / c->P) % 4 != 0 || c->K > 128 || c->cap > 1024 || c->R > 32 || c->L > 32)
    return MDR_ERR_UNSUPPORTED;
  const int A = ipow(c->K, c->P);
  if (A < 0 || A > 16384) return MDR_ERR_UNSUPPORTED;
  const int np = ipow(c->probes, c->P);
  if (np < 0 || np > 64 || np * c->cap > 4096) return MDR_ERR_UNSUPPORTED;
  if (c->dtype == MDR_BF16 && (!is_pow2_in(c->block, {64, 128}) || !is_pow2_in(c->D, {64, 128})))
    return MDR_ERR_UNSUPPORTED;
  if (c->S / c->block > 32768) return MDR_ERR_UNSUPPORTED;
  const long long tokens = static_cast<long long>(c->B) * c->S;
  if (tokens * (c->Hq + c->Hkv) * c->D > (1LL << 40)) return MDR_ERR_UNSUPPORTED;
  return MDR_OK;
}

struct Layout {
  size_t status, qrot, krot, qbar, qcodes, total;
};

Layout layout_of(const mdr_config* c) {
  const size_t nb = c->S / c->block;
  const size_t tok = static_cast<size_t>(c->B) * c->S;
  Layout l{};
  size_t o = 0;
  l.status = o; o += align_up(kStatusBytes);
  l.qrot = o;   o += align_up(tok * c->Hq * c->D * esize(c));
  l.krot = o;   o += align_up(tok * c->Hkv * c->D * esize(c));
  l.qbar = o;   o += align_up(static_cast<size_t>(c->B) * c->Hq * nb * c->D * sizeof(float));
  l.qcodes = o; o += align_up(static_cast<size_t>(c->B) * c->Hq * nb * c->P * c->probes * sizeof(int32_t));
  l.total = o;
  return l;
}

// Decode workspace: the status word and the per-(b, hq) counters of
// finished blocks (zeroed together at the start of every step), the step's
// rotated queries and per-block partial results, then (for
// mdr_decode_prefill) the rotated keys, summaries and addresses of the prefix
// at the prefix's own strides before they are copied into the state's rows.
struct DecodeLayout {
  size_t status, done, head, qrot, part, krot, kbar, addr, total;
};

DecodeLayout decode_layout_of(const mdr_config* c) {
  const size_t nb = c->S / c->block, bq = static_cast<size_t>(c->B) * c->Hq;
  DecodeLayout l{};
  size_t o = 0;
  l.status = o;
  l.done = 16;
  l.head = 16 + bq * sizeof(int32_t);                 // bytes zeroed per step
  o += align_up(l.head);
  l.qrot = o;   o += align_up(bq * c->D * sizeof(float));
  l.part = o;   o += align_up(bq * (c->R + c->L) * (2 + c->D) * sizeof(float));
  l.krot = o;   o += align_up(static_cast<size_t>(c->B) * c->S * c->Hkv * c->D * esize(c));
  l.kbar = o;   o += align_up(static_cast<size_t>(c->B) * c->Hkv * nb * c->D * sizeof(float));
  l.addr = o;   o += align_up(static_cast<size_t>(c->B) * c->Hkv * nb * sizeof(int32_t));
  l.total = o;
  return l;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(ws) + off); }

mdr_status check_ws(const mdr_config* c, void* ws, size_t ws_bytes) {
  if (!ws) return MDR_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return MDR_ERR_WORKSPACE;
  if (ws_bytes < layout_of(c).total) return MDR_ERR_WORKSPACE;
  return MDR_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

mdr_status check_index(const mdr_index* idx) {
  if (!idx || !idx->kbar || !idx->addr || !idx->lists || !idx->load || !idx->overflow || !idx->maxload)
    return MDR_ERR_INVALID_ARG;
  return MDR_OK;
}

void fill_common(SummarizeArgs& a, const mdr_config* c, const float* codebooks) {
  mdr::detail::fill_summarize_common(a, c, codebooks);
}

mdr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MDR_OK : MDR_ERR_CUDA; }

#define MDR_TRY(x)                       \
  do {                                   \
    mdr_status s_ = (x);                 \
    if (s_ != MDR_OK) return s_;         \
  } while (0)

#define MDR_CUDA(x) MDR_TRY(cuda_status(x))

// The list, route and attention steps over query / key blocks j0 .. j1 - 1
// (j1 = 0: every block).
mdr_status run_lists(const mdr_config* c, const mdr_index* idx, cudaStream_t st, int j0 = 0, int j1 = 0) {
  mdr::ListsArgs la{};
  la.addr = idx->addr; la.lists = idx->lists; la.load = idx->load;
  la.overflow = idx->overflow; la.maxload = idx->maxload;
  la.B = c->B; la.H = c->Hkv; la.nb = c->S / c->block; la.A = ipow(c->K, c->P); la.cap = c->cap;
  la.j0 = j0; la.j1 = j1;
  return cuda_status(mdr::launch_lists(la, st));
}

mdr_status run_route(const mdr_config* c, const float* qbar, const int32_t* qcodes,
                     const mdr_index* idx, int32_t* sel, int32_t* ncand, cudaStream_t st,
                     const int32_t* force = nullptr, int j0 = 0, int j1 = 0) {
  mdr::RouteArgs ra = mdr::detail::route_args(c, qbar, qcodes, idx, sel, ncand, force);
  ra.j0 = j0; ra.nbr = j1 > 0 ? j1 - j0 : 0;
  return cuda_status(mdr::launch_route(ra, st));
}

mdr_status run_attend(const mdr_config* c, const void* qrot, const void* krot, const void* v,
                      const int32_t* sel, void* out, int32_t* status, cudaStream_t st, int j0 = 0, int j1 = 0,
                      float* lse = nullptr) {
  mdr::AttendArgs aa{};
  aa.lse = lse;
  aa.j0 = j0; aa.nbr = j1 > 0 ? j1 - j0 : 0;
  aa.q = qrot; aa.k = krot; aa.v = v; aa.sel = sel; aa.out = out; aa.status = status;
  aa.tile_counter = status + 2;
  aa.B = c->B; aa.S = c->S; aa.Hq = c->Hq; aa.Hkv = c->Hkv; aa.D = c->D; aa.bs = c->block;
  aa.nb = c->S / c->block; aa.nsel = c->R + c->L;
  aa.scale = mdr::detail::softmax_scale(c);
  if (c->dtype == MDR_BF16) return cuda_status(mdr::launch_attend_tc(aa, st));
  return cuda_status(mdr::launch_attend_simt(aa, false, st));
}

}  // namespace

extern "C" {

int32_t mdr_abi_version(void) { return MDR_ABI_VERSION; }

const char* mdr_status_string(mdr_status s) {
  switch (s) {
    case MDR_OK: return "ok";
    case MDR_ERR_INVALID_ARG: return "invalid argument";
    case MDR_ERR_UNSUPPORTED: return "unsupported configuration";
    case MDR_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case MDR_ERR_CUDA: return "CUDA error";
    case MDR_ERR_DEVICE: return "device-side check failed";
  }
  return "unknown status";
}

mdr_status mdr_check_config(const mdr_config* cfg) { return check(cfg); }

mdr_status mdr_workspace_bytes(const mdr_config* cfg, size_t* bytes) {
  MDR_TRY(check(cfg));
  if (!bytes) return MDR_ERR_INVALID_ARG;
  *bytes = layout_of(cfg).total;
  return MDR_OK;
}

mdr_status mdr_build_index(const mdr_config* cfg, const void* k, const float* codebooks,
                           const mdr_index* idx, void* ws, size_t ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  if (!k || !codebooks || !aligned16(k)) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_index(idx));
  MDR_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout l = layout_of(cfg);
  MDR_CUDA(cudaMemsetAsync(at<int32_t>(ws, l.status), 0, sizeof(int32_t), st));
  SummarizeArgs a;
  fill_common(a, cfg, codebooks);
  a.x[1] = k; a.xbar[1] = idx->kbar; a.addr = idx->addr;
  a.lists_fill = idx->lists;
  a.lists_per_seq = static_cast<size_t>(cfg->Hkv) * ipow(cfg->K, cfg->P) * cfg->cap;
  a.status = at<int32_t>(ws, l.status);
  MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, st));
  return run_lists(cfg, idx, st);
}

static mdr_status route_impl(const mdr_config* cfg, const void* q, const float* codebooks,
                             const mdr_index* idx, const int32_t* force, const mdr_route_out* rt,
                             void* ws, size_t ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  if (!q || !codebooks || !rt || !rt->sel || !aligned16(q)) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_index(idx));
  MDR_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout l = layout_of(cfg);
  float* qbar = rt->qbar ? rt->qbar : at<float>(ws, l.qbar);
  int32_t* qcodes = rt->qcodes ? rt->qcodes : at<int32_t>(ws, l.qcodes);
  MDR_CUDA(cudaMemsetAsync(at<int32_t>(ws, l.status), 0, sizeof(int32_t), st));
  SummarizeArgs a;
  fill_common(a, cfg, codebooks);
  a.x[0] = q; a.xbar[0] = qbar; a.qcodes = qcodes;
  a.status = at<int32_t>(ws, l.status);
  MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, st));
  return run_route(cfg, qbar, qcodes, idx, rt->sel, rt->ncand, st, force);
}

mdr_status mdr_route(const mdr_config* cfg, const void* q, const float* codebooks,
                     const mdr_index* idx, const mdr_route_out* rt, void* ws, size_t ws_bytes,
                     void* stream) {
  return route_impl(cfg, q, codebooks, idx, nullptr, rt, ws, ws_bytes, stream);
}

mdr_status mdr_route_forced(const mdr_config* cfg, const void* q, const float* codebooks,
                            const mdr_index* idx, const int32_t* force, const mdr_route_out* rt,
                            void* ws, size_t ws_bytes, void* stream) {
  if (!force) return MDR_ERR_INVALID_ARG;
  return route_impl(cfg, q, codebooks, idx, force, rt, ws, ws_bytes, stream);
}

mdr_status mdr_target_hits(const mdr_config* cfg, const int32_t* sel, const int32_t* target,
                           int32_t* hit, int32_t* counts, void* stream) {
  MDR_TRY(check(cfg));
  if (!sel || !target || !counts) return MDR_ERR_INVALID_ARG;
  mdr::HitsArgs ha{};
  ha.sel = sel; ha.target = target; ha.hit = hit; ha.counts = counts;
  ha.nroutes = static_cast<long long>(cfg->B) * cfg->Hq * (cfg->S / cfg->block);
  ha.nsel = cfg->R + cfg->L;
  return cuda_status(mdr::launch_hits(ha, static_cast<cudaStream_t>(stream)));
}

static mdr_status attend_impl(const mdr_config* cfg, const void* q, const void* k, const void* v,
                              const int32_t* sel, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  if (!q || !k || !v || !sel || !out) return MDR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Layout l = layout_of(cfg);
  int32_t* status = at<int32_t>(ws, l.status);
  MDR_CUDA(cudaMemsetAsync(status, 0, kStatusBytes, st));
  SummarizeArgs a;
  fill_common(a, cfg, nullptr);
  a.x[0] = q; a.x[1] = k;
  a.xrot[0] = at<void>(ws, l.qrot); a.xrot[1] = at<void>(ws, l.krot);
  a.status = status;
  MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, st));
  return run_attend(cfg, at<void>(ws, l.qrot), at<void>(ws, l.krot), v, sel, out, status, st, 0, 0, lse);
}

mdr_status mdr_attend(const mdr_config* cfg, const void* q, const void* k, const void* v,
                      const int32_t* sel, void* out, void* ws, size_t ws_bytes, void* stream) {
  return attend_impl(cfg, q, k, v, sel, out, nullptr, ws, ws_bytes, stream);
}

mdr_status mdr_attend_train(const mdr_config* cfg, const void* q, const void* k, const void* v,
                            const int32_t* sel, void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!lse) return MDR_ERR_INVALID_ARG;
  return attend_impl(cfg, q, k, v, sel, out, lse, ws, ws_bytes, stream);
}

static mdr_status forward_impl(const mdr_config* cfg, const void* q, const void* k, const void* v,
                               const float* codebooks, const mdr_index* idx, const mdr_route_out* rt,
                               void* out, void* ws, size_t ws_bytes, void* stream,
                               void* const* events, int32_t n_events, float* lse = nullptr) {
  MDR_TRY(check(cfg));
  if (!q || !k || !v || !codebooks || !out || !rt || !rt->sel) return MDR_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MDR_ERR_INVALID_ARG;
  if (n_events < 0 || (n_events > 0 && !events)) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_index(idx));
  MDR_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> mdr_status {
    if (i < n_events && events[i])
      return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st));
    return MDR_OK;
  };
  const Layout l = layout_of(cfg);
  int32_t* status = at<int32_t>(ws, l.status);
  float* qbar = rt->qbar ? rt->qbar : at<float>(ws, l.qbar);
  int32_t* qcodes = rt->qcodes ? rt->qcodes : at<int32_t>(ws, l.qcodes);
  MDR_CUDA(cudaMemsetAsync(status, 0, kStatusBytes, st));
  SummarizeArgs a;
  fill_common(a, cfg, codebooks);
  a.x[0] = q; a.x[1] = k;
  a.xrot[0] = at<void>(ws, l.qrot); a.xrot[1] = at<void>(ws, l.krot);
  a.xbar[0] = qbar; a.xbar[1] = idx->kbar;
  a.qcodes = qcodes; a.addr = idx->addr;
  a.lists_fill = idx->lists;
  a.lists_per_seq = static_cast<size_t>(cfg->Hkv) * ipow(cfg->K, cfg->P) * cfg->cap;
  a.status = status;
  MDR_TRY(mark(0));
  MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, st));
  MDR_TRY(mark(1));
  MDR_TRY(run_lists(cfg, idx, st));
  MDR_TRY(mark(2));
  MDR_TRY(run_route(cfg, qbar, qcodes, idx, rt->sel, rt->ncand, st));
  MDR_TRY(mark(3));
  MDR_TRY(run_attend(cfg, at<void>(ws, l.qrot), at<void>(ws, l.krot), v, rt->sel, out, status, st, 0, 0, lse));
  return mark(4);
}

mdr_status mdr_forward(const mdr_config* cfg, const void* q, const void* k, const void* v,
                       const float* codebooks, const mdr_index* idx, const mdr_route_out* rt,
                       void* out, void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(cfg, q, k, v, codebooks, idx, rt, out, ws, ws_bytes, stream, nullptr, 0);
}

mdr_status mdr_forward_train(const mdr_config* cfg, const void* q, const void* k, const void* v,
                             const float* codebooks, const mdr_index* idx, const mdr_route_out* rt,
                             void* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!lse) return MDR_ERR_INVALID_ARG;
  return forward_impl(cfg, q, k, v, codebooks, idx, rt, out, ws, ws_bytes, stream, nullptr, 0, lse);
}

mdr_status mdr_forward_profiled(const mdr_config* cfg, const void* q, const void* k, const void* v,
                                const float* codebooks, const mdr_index* idx, const mdr_route_out* rt,
                                void* out, void* ws, size_t ws_bytes, void* stream,
                                void* const* events, int32_t n_events) {
  return forward_impl(cfg, q, k, v, codebooks, idx, rt, out, ws, ws_bytes, stream, events, n_events);
}

namespace {
struct HostLayout {
  size_t dev, q, k, v, cb, out, sel, kbar, addr, lists, load, ovf, maxl, total;
};
HostLayout host_layout_of(const mdr_config* c) {
  HostLayout h{};
  const size_t nb = c->S / c->block, tok = static_cast<size_t>(c->B) * c->S;
  const size_t A = static_cast<size_t>(ipow(c->K, c->P));
  size_t o = 0;
  h.dev = o;   o += align_up(layout_of(c).total);
  h.q = o;     o += align_up(tok * c->Hq * c->D * esize(c));
  h.k = o;     o += align_up(tok * c->Hkv * c->D * esize(c));
  h.v = o;     o += align_up(tok * c->Hkv * c->D * esize(c));
  h.cb = o;    o += align_up(static_cast<size_t>(c->K) * c->D * sizeof(float));
  h.out = o;   o += align_up(tok * c->Hq * c->D * esize(c));
  h.sel = o;   o += align_up(static_cast<size_t>(c->B) * c->Hq * nb * (c->R + c->L) * sizeof(int32_t));
  h.kbar = o;  o += align_up(static_cast<size_t>(c->B) * c->Hkv * nb * c->D * sizeof(float));
  h.addr = o;  o += align_up(static_cast<size_t>(c->B) * c->Hkv * nb * sizeof(int32_t));
  h.lists = o; o += align_up(static_cast<size_t>(c->B) * c->Hkv * A * c->cap * sizeof(int32_t));
  h.load = o;  o += align_up(static_cast<size_t>(c->B) * c->Hkv * A * sizeof(int32_t));
  h.ovf = o;   o += align_up(static_cast<size_t>(c->B) * c->Hkv * sizeof(int32_t));
  h.maxl = o;  o += align_up(static_cast<size_t>(c->B) * c->Hkv * sizeof(int32_t));
  h.total = o;
  return h;
}

// Streams and events of one mdr_forward_host call: the input copies run on
// `in`, the kernels on the caller's stream, the output copies on `out`, so
// that chunk c's output copy overlaps chunk c+1's input copy (the link is
// full duplex).
// Created on a device's first call and kept (one set per device; calls on a
// device hold its mutex, so they run one at a time).
struct HostPipeline {
  // Four chunks: each more chunk costs ~20 us of launches and waits, each
  // fewer makes the last chunk's output copy, which nothing overlaps, longer
  // (32K workload on B200: 4.40 ms with 4 chunks, 4.49 with 8, 4.66 with 16;
  // the input copy alone takes 3.66 ms at 55 GB/s).
  static constexpr int kMaxChunks = 4;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, in_done[kMaxChunks] = {}, comp_done[kMaxChunks] = {};
  bool ready = false;
  std::mutex mu;
  cudaError_t create() {
    if (ready) return cudaSuccess;
    cudaError_t e;
    if ((e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaEventCreateWithFlags(&start, cudaEventDisableTiming)) != cudaSuccess) return e;
    for (int c = 0; c < kMaxChunks; ++c) {
      if ((e = cudaEventCreateWithFlags(&in_done[c], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&comp_done[c], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    ready = true;
    return cudaSuccess;
  }
  // The copies start after whatever the caller enqueued before.  Streams
  // and events made in a context the caller has since reset are made anew.
  cudaError_t begin(cudaStream_t st) {
    cudaError_t e = create();
    if (e == cudaSuccess) e = cudaEventRecord(start, st);
    if (e == cudaErrorInvalidResourceHandle || e == cudaErrorContextIsDestroyed) {
      (void)cudaGetLastError();
      in = out = nullptr;                          // the old handles died with their context
      start = nullptr;
      for (int c = 0; c < kMaxChunks; ++c) in_done[c] = comp_done[c] = nullptr;
      ready = false;
      if ((e = create()) == cudaSuccess) e = cudaEventRecord(start, st);
    }
    if (e != cudaSuccess) return e;
    if ((e = cudaStreamWaitEvent(in, start, 0)) != cudaSuccess) return e;
    return cudaStreamWaitEvent(out, start, 0);
  }
  // Waits for the three streams.
  cudaError_t finish(cudaStream_t st) {
    cudaError_t r = cudaSuccess, e;
    if (ready && (e = cudaStreamSynchronize(in)) != cudaSuccess) r = e;
    if ((e = cudaStreamSynchronize(st)) != cudaSuccess && r == cudaSuccess) r = e;
    if (ready && (e = cudaStreamSynchronize(out)) != cudaSuccess && r == cudaSuccess) r = e;
    return r;
  }
};

HostPipeline* host_pipeline(int device) {
  constexpr int kMaxDevices = 64;
  static HostPipeline pipes[kMaxDevices];
  return device >= 0 && device < kMaxDevices ? &pipes[device] : nullptr;
}

// Rows t0 .. t1 - 1 of every sequence of a [B,S,...] tensor with row_bytes
// per token, one strided copy.
cudaError_t copy_rows(void* dst, const void* src, size_t row_bytes, int B, int S, int t0, int t1,
                      cudaMemcpyKind kind, cudaStream_t st) {
  const size_t pitch = row_bytes * S, off = row_bytes * t0;
  return cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch, static_cast<const char*>(src) + off, pitch,
                           row_bytes * (t1 - t0), B, kind, st);
}

}  // namespace

// The forward is causal: query block j's output needs the inputs of blocks
// <= j only (its summary, the index of key blocks <= j, the K/V of its
// selected blocks), and the posting lists of blocks < j are the same whether
// or not later blocks exist (each list keeps its first cap blocks in
// ascending order).  So the sequence runs in chunks of query blocks: chunk
// c's inputs are copied in, its blocks summarised, appended to the lists,
// routed and attended, and its output copied out while chunk c+1 comes in.
// The result is bit-identical to mdr_forward on the whole sequence.
static mdr_status forward_host_chunked(const mdr_config* cfg, const HostLayout& h, const void* q_host,
                                       const void* k_host, const void* v_host, const float* codebooks_host,
                                       void* out_host, int32_t* sel_host, int32_t* overflow_host,
                                       int32_t* maxload_host, void* dev_ws, cudaStream_t st, HostPipeline& pl) {
  const int nb = cfg->S / cfg->block, nsel = cfg->R + cfg->L;
  const size_t es = esize(cfg);
  const size_t qrow = static_cast<size_t>(cfg->Hq) * cfg->D * es, krow = static_cast<size_t>(cfg->Hkv) * cfg->D * es;
  const int nchunk = nb < HostPipeline::kMaxChunks ? nb : HostPipeline::kMaxChunks;
  const Layout l = layout_of(cfg);
  void* ws = at<void>(dev_ws, h.dev);
  int32_t* status = at<int32_t>(ws, l.status);
  float* qbar = at<float>(ws, l.qbar);
  int32_t* qcodes = at<int32_t>(ws, l.qcodes);
  void *q = at<void>(dev_ws, h.q), *k = at<void>(dev_ws, h.k), *v = at<void>(dev_ws, h.v);
  void* out = at<void>(dev_ws, h.out);
  const float* cb = at<float>(dev_ws, h.cb);
  mdr_index idx{at<float>(dev_ws, h.kbar), at<int32_t>(dev_ws, h.addr), at<int32_t>(dev_ws, h.lists),
                at<int32_t>(dev_ws, h.load), at<int32_t>(dev_ws, h.ovf), at<int32_t>(dev_ws, h.maxl)};
  int32_t* sel = at<int32_t>(dev_ws, h.sel);
  const size_t lists_bytes = static_cast<size_t>(cfg->B) * cfg->Hkv * ipow(cfg->K, cfg->P) * cfg->cap * sizeof(int32_t);

  MDR_CUDA(cudaMemcpyAsync(at<void>(dev_ws, h.cb), codebooks_host, static_cast<size_t>(cfg->K) * cfg->D * sizeof(float),
                           cudaMemcpyHostToDevice, pl.in));
  MDR_CUDA(cudaMemsetAsync(status, 0, kStatusBytes, st));
  MDR_CUDA(cudaMemsetAsync(idx.lists, 0xff, lists_bytes, st));   // every list empty (-1)
  for (int c = 0; c < nchunk; ++c) {
    // Decreasing chunks (4, 3, 2, 1 tenths of the blocks): the last chunk's
    // kernels and output copy, which nothing overlaps, are the shortest
    // (32K workload: 4.25 ms per call against 4.79 with equal chunks).
    static constexpr int kEdge[5] = {0, 4, 7, 9, 10};
    const int j0 = nchunk == 4 ? static_cast<int>(static_cast<long long>(nb) * kEdge[c] / 10)
                               : static_cast<int>(static_cast<long long>(nb) * c / nchunk);
    const int j1 = nchunk == 4 ? static_cast<int>(static_cast<long long>(nb) * kEdge[c + 1] / 10)
                               : static_cast<int>(static_cast<long long>(nb) * (c + 1) / nchunk);
    if (j1 <= j0) continue;
    const int t0 = j0 * cfg->block, t1 = j1 * cfg->block;
    MDR_CUDA(copy_rows(q, q_host, qrow, cfg->B, cfg->S, t0, t1, cudaMemcpyHostToDevice, pl.in));
    MDR_CUDA(copy_rows(k, k_host, krow, cfg->B, cfg->S, t0, t1, cudaMemcpyHostToDevice, pl.in));
    MDR_CUDA(copy_rows(v, v_host, krow, cfg->B, cfg->S, t0, t1, cudaMemcpyHostToDevice, pl.in));
    MDR_CUDA(cudaEventRecord(pl.in_done[c], pl.in));
    MDR_CUDA(cudaStreamWaitEvent(st, pl.in_done[c], 0));
    MDR_CUDA(cudaMemsetAsync(status + 2, 0, sizeof(int32_t), st));   // the attention's tile counter
    SummarizeArgs a;
    fill_common(a, cfg, cb);
    a.x[0] = q; a.x[1] = k;
    a.xrot[0] = at<void>(ws, l.qrot); a.xrot[1] = at<void>(ws, l.krot);
    a.xbar[0] = qbar; a.xbar[1] = idx.kbar;
    a.qcodes = qcodes; a.addr = idx.addr;
    a.status = status;
    a.j0 = j0; a.nbr = j1 - j0;
    MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, st));
    MDR_TRY(run_lists(cfg, &idx, st, j0, j1));
    MDR_TRY(run_route(cfg, qbar, qcodes, &idx, sel, nullptr, st, nullptr, j0, j1));
    MDR_TRY(run_attend(cfg, at<void>(ws, l.qrot), at<void>(ws, l.krot), v, sel, out, status, st, j0, j1));
    MDR_CUDA(cudaEventRecord(pl.comp_done[c], st));
    MDR_CUDA(cudaStreamWaitEvent(pl.out, pl.comp_done[c], 0));
    MDR_CUDA(copy_rows(out_host, out, qrow, cfg->B, cfg->S, t0, t1, cudaMemcpyDeviceToHost, pl.out));
    if (sel_host) {
      const size_t row = static_cast<size_t>(nsel) * sizeof(int32_t);
      MDR_CUDA(cudaMemcpy2DAsync(sel_host + static_cast<size_t>(j0) * nsel, nb * row, sel + static_cast<size_t>(j0) * nsel,
                                 nb * row, (j1 - j0) * row, static_cast<size_t>(cfg->B) * cfg->Hq,
                                 cudaMemcpyDeviceToHost, pl.out));
    }
  }
  const size_t bh = static_cast<size_t>(cfg->B) * cfg->Hkv * sizeof(int32_t);
  if (overflow_host) MDR_CUDA(cudaMemcpyAsync(overflow_host, idx.overflow, bh, cudaMemcpyDeviceToHost, pl.out));
  if (maxload_host) MDR_CUDA(cudaMemcpyAsync(maxload_host, idx.maxload, bh, cudaMemcpyDeviceToHost, pl.out));
  return MDR_OK;
}


mdr_status mdr_host_workspace_bytes(const mdr_config* cfg, size_t* bytes) {
  MDR_TRY(check(cfg));
  if (!bytes) return MDR_ERR_INVALID_ARG;
  *bytes = host_layout_of(cfg).total;
  return MDR_OK;
}

mdr_status mdr_forward_host(const mdr_config* cfg, const void* q_host, const void* k_host,
                            const void* v_host, const float* codebooks_host, void* out_host,
                            int32_t* sel_host, int32_t* overflow_host, int32_t* maxload_host,
                            void* dev_ws, size_t dev_ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  if (!q_host || !k_host || !v_host || !codebooks_host || !out_host) return MDR_ERR_INVALID_ARG;
  const HostLayout h = host_layout_of(cfg);
  if (!dev_ws || reinterpret_cast<uintptr_t>(dev_ws) % kAlign != 0 || dev_ws_bytes < h.total)
    return MDR_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int device = -1;
  MDR_CUDA(cudaGetDevice(&device));
  HostPipeline* pl = host_pipeline(device);
  if (!pl) return MDR_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(pl->mu);
  MDR_CUDA(pl->begin(st));
  const mdr_status s = forward_host_chunked(cfg, h, q_host, k_host, v_host, codebooks_host, out_host, sel_host,
                                            overflow_host, maxload_host, dev_ws, st, *pl);
  // Whatever was enqueued finishes before the call returns.
  const cudaError_t e = pl->finish(st);
  MDR_TRY(s);
  MDR_CUDA(e);
  int32_t code = 0;
  MDR_CUDA(cudaMemcpy(&code, at<int32_t>(dev_ws, h.dev), sizeof(int32_t), cudaMemcpyDeviceToHost));
  return code == 0 ? MDR_OK : MDR_ERR_DEVICE;
}

mdr_status mdr_read_device_status(const void* ws, int32_t* code, void* stream) {
  if (!ws || !code) return MDR_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MDR_CUDA(cudaStreamSynchronize(st));
  MDR_CUDA(cudaMemcpy(code, ws, sizeof(int32_t), cudaMemcpyDeviceToHost));
  return *code == 0 ? MDR_OK : MDR_ERR_DEVICE;
}


// ------------------------------------------------------------------ decoding
static mdr_status check_decode_state(const mdr_decode_state* st) {
  if (!st || !st->krot || !st->v || !st->ksum) return MDR_ERR_INVALID_ARG;
  if (!aligned16(st->krot) || !aligned16(st->v) || !aligned16(st->ksum) || !aligned16(st->idx.kbar))
    return MDR_ERR_INVALID_ARG;
  return check_index(&st->idx);
}

static mdr_status check_decode_ws(const mdr_config* c, void* ws, size_t ws_bytes) {
  if (!ws || reinterpret_cast<uintptr_t>(ws) % kAlign != 0) return MDR_ERR_WORKSPACE;
  if (ws_bytes < decode_layout_of(c).total) return MDR_ERR_WORKSPACE;
  return MDR_OK;
}

mdr_status mdr_decode_workspace_bytes(const mdr_config* cfg, size_t* bytes) {
  MDR_TRY(check(cfg));
  if (!bytes) return MDR_ERR_INVALID_ARG;
  *bytes = decode_layout_of(cfg).total;
  return MDR_OK;
}

mdr_status mdr_decode_reset(const mdr_config* cfg, const mdr_decode_state* st, void* stream) {
  MDR_TRY(check(cfg));
  MDR_TRY(check_decode_state(st));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bh = static_cast<size_t>(cfg->B) * cfg->Hkv, A = static_cast<size_t>(ipow(cfg->K, cfg->P));
  const size_t nb = cfg->S / cfg->block;
  MDR_CUDA(cudaMemsetAsync(st->idx.lists, 0xff, bh * A * cfg->cap * sizeof(int32_t), s));
  MDR_CUDA(cudaMemsetAsync(st->idx.addr, 0xff, bh * nb * sizeof(int32_t), s));
  MDR_CUDA(cudaMemsetAsync(st->idx.load, 0, bh * A * sizeof(int32_t), s));
  MDR_CUDA(cudaMemsetAsync(st->idx.overflow, 0, bh * sizeof(int32_t), s));
  MDR_CUDA(cudaMemsetAsync(st->idx.maxload, 0, bh * sizeof(int32_t), s));
  MDR_CUDA(cudaMemsetAsync(st->ksum, 0, bh * cfg->D * sizeof(float), s));
  return MDR_OK;
}

mdr_status mdr_decode_prefill(const mdr_config* cfg, int32_t S0, const void* k, const void* v,
                              const float* codebooks, const mdr_decode_state* st, void* ws,
                              size_t ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  MDR_TRY(check_decode_state(st));
  if (S0 < 0 || S0 > cfg->S || S0 % cfg->block != 0) return MDR_ERR_INVALID_ARG;
  if (S0 > 0 && (!k || !v || !codebooks || !aligned16(k) || !aligned16(v))) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_decode_ws(cfg, ws, ws_bytes));
  MDR_TRY(mdr_decode_reset(cfg, st, stream));
  if (S0 == 0) return MDR_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DecodeLayout l = decode_layout_of(cfg);
  int32_t* status = at<int32_t>(ws, l.status);
  MDR_CUDA(cudaMemsetAsync(status, 0, sizeof(int32_t), s));
  mdr_config c0 = *cfg;
  c0.S = S0;
  const size_t nb = cfg->S / cfg->block, nb0 = S0 / cfg->block, e = esize(cfg);
  const size_t rows_k = static_cast<size_t>(cfg->Hkv) * cfg->D * e;          // bytes of one token's keys
  // The prefix's rows land in place when the strides agree; else in the
  // workspace, then copied.
  const bool k_in_place = cfg->B == 1 || S0 == cfg->S;
  const bool kbar_in_place = static_cast<size_t>(cfg->B) * cfg->Hkv == 1 || nb0 == nb;
  void* krot0 = k_in_place ? st->krot : at<void>(ws, l.krot);
  float* kbar0 = kbar_in_place ? st->idx.kbar : at<float>(ws, l.kbar);
  int32_t* addr0 = kbar_in_place ? st->idx.addr : at<int32_t>(ws, l.addr);
  SummarizeArgs a;
  fill_common(a, &c0, codebooks);
  a.x[1] = k; a.xrot[1] = krot0; a.xbar[1] = kbar0; a.addr = addr0;
  a.lists_fill = st->idx.lists;
  a.lists_per_seq = static_cast<size_t>(cfg->Hkv) * ipow(cfg->K, cfg->P) * cfg->cap;
  a.status = status;
  MDR_CUDA(mdr::launch_summarize(a, cfg->dtype == MDR_BF16, s));
  mdr_index idx0 = st->idx;
  idx0.kbar = kbar0;
  idx0.addr = addr0;
  MDR_TRY(run_lists(&c0, &idx0, s));
  if (!k_in_place)
    MDR_CUDA(cudaMemcpy2DAsync(st->krot, cfg->S * rows_k, krot0, S0 * rows_k, S0 * rows_k, cfg->B,
                               cudaMemcpyDeviceToDevice, s));
  MDR_CUDA(cudaMemcpy2DAsync(st->v, cfg->S * rows_k, v, S0 * rows_k, S0 * rows_k, cfg->B,
                             cudaMemcpyDeviceToDevice, s));
  if (!kbar_in_place) {
    const size_t bh = static_cast<size_t>(cfg->B) * cfg->Hkv;
    MDR_CUDA(cudaMemcpy2DAsync(st->idx.kbar, nb * cfg->D * sizeof(float), kbar0, nb0 * cfg->D * sizeof(float),
                               nb0 * cfg->D * sizeof(float), bh, cudaMemcpyDeviceToDevice, s));
    MDR_CUDA(cudaMemcpy2DAsync(st->idx.addr, nb * sizeof(int32_t), addr0, nb0 * sizeof(int32_t),
                               nb0 * sizeof(int32_t), bh, cudaMemcpyDeviceToDevice, s));
  }
  return MDR_OK;
}

mdr_status mdr_decode_step(const mdr_config* cfg, int32_t t, const void* q_t, const void* k_t,
                           const void* v_t, const float* codebooks, const mdr_decode_state* st,
                           void* out_t, int32_t* sel_t, int32_t* ncand_t, void* ws, size_t ws_bytes,
                           void* stream) {
  MDR_TRY(check(cfg));
  MDR_TRY(check_decode_state(st));
  if (t < 0 || t >= cfg->S) return MDR_ERR_INVALID_ARG;
  if (!q_t || !k_t || !v_t || !codebooks || !out_t || !sel_t || !aligned16(codebooks)) return MDR_ERR_INVALID_ARG;
  MDR_TRY(check_decode_ws(cfg, ws, ws_bytes));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const DecodeLayout l = decode_layout_of(cfg);
  MDR_CUDA(cudaMemsetAsync(ws, 0, l.head, s));
  mdr::DecodeArgs d;
  std::memset(&d, 0, sizeof(d));
  d.t = t; d.q_t = q_t; d.k_t = k_t; d.v_t = v_t;
  d.krot = st->krot; d.v = st->v; d.ksum = st->ksum;
  d.kbar = st->idx.kbar; d.addr = st->idx.addr; d.lists = st->idx.lists; d.load = st->idx.load;
  d.overflow = st->idx.overflow; d.maxload = st->idx.maxload;
  d.codebooks = codebooks; d.out_t = out_t; d.sel_t = sel_t; d.ncand_t = ncand_t;
  d.qrot_t = at<float>(ws, l.qrot); d.part = at<float>(ws, l.part); d.done = at<int32_t>(ws, l.done);
  d.B = cfg->B; d.S = cfg->S; d.Hq = cfg->Hq; d.Hkv = cfg->Hkv; d.D = cfg->D; d.bs = cfg->block;
  d.nb = cfg->S / cfg->block; d.P = cfg->P; d.K = cfg->K; d.A = ipow(cfg->K, cfg->P); d.cap = cfg->cap;
  d.probes = cfg->probes; d.R = cfg->R; d.L = cfg->L;
  d.scale = mdr::detail::softmax_scale(cfg);
  mdr::detail::fill_inv_freq(d.inv_freq, cfg);
  return cuda_status(mdr::launch_decode(d, cfg->dtype == MDR_BF16, s));
}

// ------------------------------------------------------------------ backward
struct BwdLayout {
  size_t status, qr, kr, lse, delta, rev_off, rev, total;
};

static BwdLayout bwd_layout_of(const mdr_config* c) {
  BwdLayout l{};
  const size_t tok = static_cast<size_t>(c->B) * c->S;
  const size_t nb = static_cast<size_t>(c->S / c->block);
  size_t o = 0;
  l.status = o;  o += align_up(16);
  l.qr = o;      o += align_up(tok * c->Hq * c->D * sizeof(float));
  l.kr = o;      o += align_up(tok * c->Hkv * c->D * sizeof(float));
  l.lse = o;     o += align_up(tok * c->Hq * sizeof(float));
  l.delta = o;   o += align_up(tok * c->Hq * sizeof(float));
  l.rev_off = o; o += align_up(static_cast<size_t>(c->B) * c->Hkv * (nb + 1) * sizeof(int32_t));
  l.rev = o;     o += align_up(static_cast<size_t>(c->B) * c->Hq * nb * (c->R + c->L) * sizeof(int32_t));
  l.total = o;
  return l;
}

mdr_status mdr_backward_workspace_bytes(const mdr_config* cfg, size_t* bytes) {
  MDR_TRY(check(cfg));
  if (!bytes) return MDR_ERR_INVALID_ARG;
  *bytes = bwd_layout_of(cfg).total;
  return MDR_OK;
}

static mdr_status backward_impl(const mdr_config* cfg, const void* q, const void* k, const void* v,
                                const int32_t* sel, const void* out, const float* lse, const void* dout,
                                float* dq, float* dk, float* dv, void* ws, size_t ws_bytes, void* stream) {
  MDR_TRY(check(cfg));
  if (!q || !k || !v || !sel || !dout || !dq || !dk || !dv) return MDR_ERR_INVALID_ARG;
  if ((out == nullptr) != (lse == nullptr)) return MDR_ERR_INVALID_ARG;
  const BwdLayout l = bwd_layout_of(cfg);
  if (!ws || reinterpret_cast<uintptr_t>(ws) % kAlign != 0 || ws_bytes < l.total) return MDR_ERR_WORKSPACE;
  if (static_cast<long long>(cfg->B) * cfg->Hq * (cfg->S / cfg->block) * (cfg->block / 16) > INT32_MAX)
    return MDR_ERR_UNSUPPORTED;
  if (mdr::bwd_rev_smem(cfg->S / cfg->block) > kMaxDynamicSmem) return MDR_ERR_UNSUPPORTED;   // reverse index
  if (static_cast<long long>(cfg->Hq / cfg->Hkv) * (cfg->S / cfg->block) * (cfg->R + cfg->L) > INT32_MAX)
    return MDR_ERR_UNSUPPORTED;                                 // reverse-index entries of one KV head
  const bool tc = cfg->dtype == MDR_BF16;          // tensor cores (block and D in {64,128} for bf16)
  if (tc && (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
             !aligned16(dk) || !aligned16(dv)))
    return MDR_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the status word and, for the tensor-core kernels, where a CTA gave up
  MDR_CUDA(cudaMemsetAsync(at<int32_t>(ws, l.status), 0, 4 * sizeof(int32_t), st));
  mdr::BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.q = q; a.k = k; a.v = v; a.dout = dout; a.sel = sel;
  a.qr = at<float>(ws, l.qr); a.kr = at<float>(ws, l.kr);
  a.lse = at<float>(ws, l.lse); a.delta = at<float>(ws, l.delta);
  a.rev_off = at<int32_t>(ws, l.rev_off); a.rev = at<int32_t>(ws, l.rev);
  a.dq = dq; a.dk = dk; a.dv = dv; a.status = at<int32_t>(ws, l.status);
  a.B = cfg->B; a.S = cfg->S; a.Hq = cfg->Hq; a.Hkv = cfg->Hkv; a.D = cfg->D; a.bs = cfg->block;
  a.nb = cfg->S / cfg->block; a.nsel = cfg->R + cfg->L;
  a.scale = mdr::detail::softmax_scale(cfg);
  mdr::detail::fill_inv_freq(a.inv_freq, cfg);
  if (!tc) return cuda_status(mdr::launch_backward(a, false, st));   // float32 recomputes the statistics
  a.out_in = out; a.lse_in = lse;
  // The rotated copies in the storage type, by the summary kernel (the
  // operands the forward's attention reads), into the float32 regions.
  SummarizeArgs sa;
  fill_common(sa, cfg, nullptr);
  sa.x[0] = q; sa.x[1] = k;
  sa.xrot[0] = a.qr; sa.xrot[1] = a.kr;
  sa.status = a.status;
  MDR_CUDA(mdr::launch_summarize(sa, true, st));
  a.qrot = a.qr; a.krot = a.kr;
  return cuda_status(mdr::launch_backward_tc(a, st));
}

mdr_status mdr_attend_backward(const mdr_config* cfg, const void* q, const void* k, const void* v,
                               const int32_t* sel, const void* dout, float* dq, float* dk, float* dv,
                               void* ws, size_t ws_bytes, void* stream) {
  return backward_impl(cfg, q, k, v, sel, nullptr, nullptr, dout, dq, dk, dv, ws, ws_bytes, stream);
}

mdr_status mdr_attend_backward_saved(const mdr_config* cfg, const void* q, const void* k, const void* v,
                                     const int32_t* sel, const void* out, const float* lse, const void* dout,
                                     float* dq, float* dk, float* dv, void* ws, size_t ws_bytes, void* stream) {
  if (!out || !lse) return MDR_ERR_INVALID_ARG;
  if (cfg && cfg->dtype == MDR_BF16 && !aligned16(out)) return MDR_ERR_INVALID_ARG;
  return backward_impl(cfg, q, k, v, sel, out, lse, dout, dq, dk, dv, ws, ws_bytes, stream);
}

// ------------------------------------------------------ codebook calibration
struct CalibLayout {
  size_t assign, part, pcount, total;
  int chunk, nchunk, warps;
};

static mdr_status check_calib(int64_t N, int32_t D, int32_t P, int32_t K) {
  if (N < 1 || P < 1 || K < 1) return MDR_ERR_INVALID_ARG;
  if (D != 32 && D != 64 && D != 128) return MDR_ERR_UNSUPPORTED;
  if (P > 4 || D % P != 0 || (D / P) % 4 != 0 || D / P < 8 || K > 128) return MDR_ERR_UNSUPPORTED;
  if (N > INT32_MAX / P) return MDR_ERR_UNSUPPORTED;
  return MDR_OK;
}

static CalibLayout calib_layout_of(int64_t N, int32_t D, int32_t P, int32_t K) {
  CalibLayout l{};
  mdr::calib_plan(N, D, P, K, &l.chunk, &l.nchunk, &l.warps);
  size_t o = 0;
  l.assign = o; o += align_up(static_cast<size_t>(N) * P * sizeof(int32_t));
  l.part = o;   o += align_up(static_cast<size_t>(P) * l.nchunk * K * (D / P) * sizeof(float));
  l.pcount = o; o += align_up(static_cast<size_t>(P) * l.nchunk * K * sizeof(int32_t));
  l.total = o;
  return l;
}

mdr_status mdr_calibrate_workspace_bytes(int64_t N, int32_t D, int32_t P, int32_t K, size_t* bytes) {
  MDR_TRY(check_calib(N, D, P, K));
  if (!bytes) return MDR_ERR_INVALID_ARG;
  *bytes = calib_layout_of(N, D, P, K).total;
  return MDR_OK;
}

mdr_status mdr_calibrate_codebooks(const float* records, int64_t N, int32_t D, int32_t P, int32_t K,
                                   const float* codebooks_in, float* codebooks_out, int32_t rounds,
                                   int32_t* counts, int32_t* assign, void* ws, size_t ws_bytes,
                                   void* stream) {
  MDR_TRY(check_calib(N, D, P, K));
  if (!records || !codebooks_in || !codebooks_out || rounds < 0) return MDR_ERR_INVALID_ARG;
  if (!aligned16(records) || !aligned16(codebooks_in) || !aligned16(codebooks_out)) return MDR_ERR_INVALID_ARG;
  const size_t cb_bytes = static_cast<size_t>(K) * D * sizeof(float);
  const char* ci = reinterpret_cast<const char*>(codebooks_in);
  const char* co = reinterpret_cast<const char*>(codebooks_out);
  if (ci != co && ci < co + cb_bytes && co < ci + cb_bytes) return MDR_ERR_INVALID_ARG;   // partial overlap
  const CalibLayout l = calib_layout_of(N, D, P, K);
  if (!ws || reinterpret_cast<uintptr_t>(ws) % kAlign != 0 || ws_bytes < l.total) return MDR_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (rounds == 0) {
    if (ci != co) MDR_CUDA(cudaMemcpyAsync(codebooks_out, codebooks_in, cb_bytes, cudaMemcpyDeviceToDevice, st));
    return MDR_OK;
  }
  int32_t* asg = assign ? assign : at<int32_t>(ws, l.assign);
  mdr::CodesArgs ca{};
  ca.xbar[0] = records; ca.H[0] = 1; ca.qcodes = asg;
  ca.B = 1; ca.nb = static_cast<int>(N); ca.D = D; ca.P = P; ca.K = K; ca.probes = 1;
  mdr::CalibArgs a{};
  a.records = records; a.assign = asg; a.cb_new = codebooks_out;
  a.part = at<float>(ws, l.part); a.pcount = at<int32_t>(ws, l.pcount);
  a.N = N; a.D = D; a.P = P; a.K = K; a.chunk = l.chunk; a.nchunk = l.nchunk; a.warps = l.warps;
  for (int r = 0; r < rounds; ++r) {
    const float* cur = r == 0 ? codebooks_in : codebooks_out;
    ca.codebooks = cur;
    ca.codebooks_written_before = r > 0;
    MDR_CUDA(mdr::launch_codes(ca, st));
    a.cb_old = cur;
    a.counts = r == rounds - 1 ? counts : nullptr;
    MDR_CUDA(mdr::launch_calibrate_round(a, st));
  }
  return MDR_OK;
}

}  // extern "C"
