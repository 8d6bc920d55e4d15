// Argument filling shared by the C-ABI entry points (mdr_abi.cu,
// mdr_noalloc.cu): one place turns an mdr_config into the kernels' launch
// arguments, so every entry point that runs a step runs it the same way.
#pragma once

#include <cmath>
#include <cstring>

#include "mdr.h"
#include "kernels.h"

namespace mdr {
namespace detail {

// b^e, or -1 once it exceeds 2^30.
inline int ipow(int b, int e) {
  long long r = 1;
  for (int i = 0; i < e; ++i) {
    r *= b;
    if (r > (1LL << 30)) return -1;
  }
  return static_cast<int>(r);
}

// Rotary frequencies omega_i = base^(-2i/D), i < D/2: computed in double,
// rounded to float (the angle of pair i at position t is then the float32
// product t * omega_i).
inline void fill_inv_freq(float* inv_freq, const mdr_config* c) {
  for (int i = 0; i < c->D / 2; ++i)
    inv_freq[i] = static_cast<float>(std::pow(static_cast<double>(c->rope_base), -2.0 * i / c->D));
}

// Softmax scale: cfg->scale, or 1/sqrt(D) when it is 0.
inline float softmax_scale(const mdr_config* c) {
  return c->scale > 0.f ? c->scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(c->D)));
}

// Shapes, codebooks and rotary frequencies of a summary launch; the caller
// sets the sides, outputs and status word.
inline void fill_summarize_common(SummarizeArgs& a, const mdr_config* c, const float* codebooks) {
  std::memset(&a, 0, sizeof(a));
  a.H[0] = c->Hq;
  a.H[1] = c->Hkv;
  a.codebooks = codebooks;
  a.B = c->B; a.S = c->S; a.D = c->D; a.bs = c->block; a.nb = c->S / c->block;
  a.P = c->P; a.K = c->K; a.probes = c->probes;
  fill_inv_freq(a.inv_freq, c);
}

// Arguments of the route kernel over an index.
inline RouteArgs route_args(const mdr_config* c, const float* qbar, const int32_t* qcodes,
                            const mdr_index* idx, int32_t* sel, int32_t* ncand,
                            const int32_t* force = nullptr) {
  RouteArgs ra{};
  ra.qbar = qbar; ra.qcodes = qcodes; ra.kbar = idx->kbar; ra.lists = idx->lists; ra.load = idx->load;
  ra.sel = sel; ra.ncand = ncand; ra.force = force;
  ra.B = c->B; ra.Hq = c->Hq; ra.Hkv = c->Hkv; ra.nb = c->S / c->block; ra.D = c->D;
  ra.P = c->P; ra.K = c->K; ra.A = ipow(c->K, c->P); ra.probes = c->probes; ra.cap = c->cap;
  ra.R = c->R; ra.L = c->L;
  return ra;
}

}  // namespace detail
}  // namespace mdr
