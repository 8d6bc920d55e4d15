// Internal launch interface of the libmdr kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace mdr {

// Launch facts cached per device (launch_cache.cu).
int cached_sm_count();                                        // 0 on error
cudaError_t cached_allow_smem(const void* fn, int bytes);     // dynamic shared memory the kernel may use
int cached_occupancy(const void* fn, int threads, size_t smem);   // blocks per SM, 0 on error

// K1 + K2: rotate, summarise and code one or both sides.
struct SummarizeArgs {
  const void* x[2];        // side 0 = queries [B,S,Hq,D], side 1 = keys [B,S,Hkv,D]; null skips a side
  void* xrot[2];           // rotated copies (same layout and type); null = not written
  float* xbar[2];          // block means [B,H,nb,D] float32; null = not written
  int H[2];                // Hq, Hkv
  int32_t* qcodes;         // [B,Hq,nb,P,probes]; null = no query codes
  int32_t* addr;           // [B,Hkv,nb]; null = no key addresses
  const float* codebooks;  // [P,K,D/P]
  int B, S, D, bs, nb, P, K, probes;
  float inv_freq[64];      // omega_i, i < D/2
  int32_t* lists_fill;     // posting lists [B, Hkv*A*cap] padded with -1 by the key side; null = skip
  size_t lists_per_seq;    // Hkv*A*cap
  int32_t* status;         // device status word (a wait that ran out writes 1); null = none
  int j0, nbr;             // blocks j0 .. j0 + nbr - 1 only (nbr = 0: every block, j0 = 0)
};
size_t summarize_smem_bytes(int bs, int D, int Hq, int Hkv);
// Launches K1 (rotation, summaries) and, when qcodes or addr is given, K2.
cudaError_t launch_summarize(const SummarizeArgs& a, bool bf16, cudaStream_t st);

// K2: codes of the block summaries (queries: top-p per subspace; keys: address).
struct CodesArgs {
  const float* xbar[2];    // summaries [B,H,nb,D] per side; null skips a side
  int H[2];                // Hq, Hkv
  int32_t* qcodes;         // [B,Hq,nb,P,probes] (side 0)
  int32_t* addr;           // [B,Hkv,nb] (side 1)
  const float* codebooks;  // [P,K,D/P]
  int B, nb, D, P, K, probes;
  bool codebooks_written_before;   // the previous kernel on the stream writes the codebooks
  int j0, nbr;             // rows of blocks j0 .. j0 + nbr - 1 only (nbr = 0: every block)
};
cudaError_t launch_codes(const CodesArgs& a, cudaStream_t st);

// Codebook calibration, one round of spherical k-means per subspace after
// the codes kernel has assigned every record (probes = 1).
struct CalibArgs {
  const float* records;    // [N,D]
  const int32_t* assign;   // [N,P]
  const float* cb_old;     // [P,K,dsub] codebooks the round started from
  float* cb_new;           // [P,K,dsub]; may equal cb_old
  float* part;             // scratch [P,nchunk,K,dsub]
  int32_t* pcount;         // scratch [P,nchunk,K]
  int32_t* counts;         // [P,K] members per codeword, or null
  long long N;
  int D, P, K, chunk, nchunk, warps;
};
// Chunking of N records for the partial sums (records per CTA, CTAs per
// subspace, warps per CTA) and the scratch it needs.
void calib_plan(long long N, int D, int P, int K, int* chunk, int* nchunk, int* warps);
cudaError_t launch_calibrate_round(const CalibArgs& a, cudaStream_t st);

// K3: bounded causal posting lists of every (b, kv head).
struct ListsArgs {
  const int32_t* addr;     // [B,Hkv,nb]
  int32_t* lists;          // [B,Hkv,A,cap]
  int32_t* load;           // [B,Hkv,A]
  int32_t* overflow;       // [B,Hkv]
  int32_t* maxload;        // [B,Hkv]
  int B, H, nb, A, cap;
  // Blocks j0 .. j1 - 1 are added, in order.  j0 = 0 starts from empty
  // lists; j0 > 0 continues from the counts in load (the lists of blocks
  // < j0 already built).  j1 = 0: every block.
  int j0, j1;
};
cudaError_t launch_lists(const ListsArgs& a, cudaStream_t st);

// K4: probe / rerank / top-R + locals, one warp per (b, hq, j).
struct RouteArgs {
  const float* qbar;       // [B,Hq,nb,D]
  const int32_t* qcodes;   // [B,Hq,nb,P,probes]
  const float* kbar;       // [B,Hkv,nb,D]
  const int32_t* lists;    // [B,Hkv,A,cap]
  const int32_t* load;     // [B,Hkv,A]
  int32_t* sel;            // [B,Hq,nb,R+L]
  int32_t* ncand;          // [B,Hq,nb] or null
  const int32_t* force;    // [B,Hq,nb] forced target block per route (-1 none) or null
  // Status word of the kernels that wrote qbar and qcodes, or null.  When it
  // is nonzero (a bounded wait there ran out, so the summaries may be
  // incomplete) every route writes a row of -1 and ncand -1 instead of routing.
  const int32_t* upstream_status;
  int B, Hq, Hkv, nb, D, P, K, A, probes, cap, R, L;
  int j0, nbr;             // query blocks j0 .. j0 + nbr - 1 only (nbr = 0: every block)
};
cudaError_t launch_route(const RouteArgs& a, cudaStream_t st);

// Target-block hit diagnostic: per route whether its target is selected.
struct HitsArgs {
  const int32_t* sel;      // [B,Hq,nb,nsel]
  const int32_t* target;   // [B,Hq,nb], -1 = no target
  int32_t* hit;            // [B,Hq,nb]: 1 hit, 0 miss, -1 no target; or null
  int32_t* counts;         // [2]: routes with a target, hits
  long long nroutes;
  int nsel;
};
cudaError_t launch_hits(const HitsArgs& a, cudaStream_t st);

// K5: selected-set causal attention over rotated q', k' and v.
struct AttendArgs {
  const void* q;           // rotated queries [B,S,Hq,D]
  const void* k;           // rotated keys    [B,S,Hkv,D]
  const void* v;           // values          [B,S,Hkv,D]
  const int32_t* sel;      // [B,Hq,nb,R+L]
  void* out;               // [B,S,Hq,D]
  int32_t* status;         // device status word
  int32_t* tile_counter;   // tensor-core kernel: zero at launch; tiles are handed out from it
  float* lse;              // [B,Hq,S] natural-log normaliser of each row's softmax
                           // (-inf for a row with nothing selected), or null
  int B, S, Hq, Hkv, D, bs, nb, nsel;
  float scale;
  int j0, nbr;             // query blocks j0 .. j0 + nbr - 1 only (nbr = 0: every block)
};
cudaError_t launch_attend_simt(const AttendArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t st);
// Block 128 with two or more query heads per KV head: one unit per pair of
// query heads, the union of their selected blocks gathered once.
cudaError_t launch_attend_union(const AttendArgs& a, cudaStream_t st);

// K6: one decode step (token t of every sequence) on a caller-owned state.
struct DecodeArgs {
  int t;                   // position of the new token
  const void* q_t;         // [B,Hq,D]
  const void* k_t;         // [B,Hkv,D]
  const void* v_t;         // [B,Hkv,D]
  void* krot;              // state: rotated keys [B,S,Hkv,D]
  void* v;                 // state: values [B,S,Hkv,D]
  float* ksum;             // state: float32 sum of the current block's rotated keys [B,Hkv,D]
  float* kbar;             // state index [B,Hkv,nb,D]
  int32_t* addr;           // [B,Hkv,nb]
  int32_t* lists;          // [B,Hkv,A,cap]
  int32_t* load;           // [B,Hkv,A]
  int32_t* overflow;       // [B,Hkv]
  int32_t* maxload;        // [B,Hkv]
  const float* codebooks;  // [P,K,D/P]
  void* out_t;             // [B,Hq,D]
  int32_t* sel_t;          // [B,Hq,R+L]
  int32_t* ncand_t;        // [B,Hq] or null
  float* qrot_t;           // scratch: rotated queries [B,Hq,D]
  float* part;             // scratch: per selected block max, sum, output [B,Hq,R+L,2+D]
  int32_t* done;           // scratch: blocks finished per (b, hq) [B,Hq], zero at the start of a step
  int B, S, Hq, Hkv, D, bs, nb, P, K, A, cap, probes, R, L;
  float scale;
  float inv_freq[64];      // omega_i, i < D/2
};
cudaError_t launch_decode(const DecodeArgs& a, bool bf16, cudaStream_t st);

// Backward of the selected-set attention (route fixed): dq, dk, dv in float32.
struct BwdArgs {
  const void* q;           // [B,S,Hq,D] storage type (not rotated)
  const void* k;           // [B,S,Hkv,D]
  const void* v;           // [B,S,Hkv,D]
  const void* dout;        // [B,S,Hq,D] upstream gradient, storage type
  const int32_t* sel;      // [B,Hq,nb,nsel]
  float* qr;               // scratch: rotated q, float32 [B,S,Hq,D] (CUDA-core path)
  float* kr;               // scratch: rotated k, float32 [B,S,Hkv,D] (CUDA-core path)
  const void* qrot;        // rotated q in the storage type [B,S,Hq,D] (tensor-core path)
  const void* krot;        // rotated k in the storage type [B,S,Hkv,D] (tensor-core path)
  float* lse;              // scratch: [B,Hq,S] log-sum-exp of the scaled scores
  float* delta;            // scratch: [B,Hq,S] dout_t . out_t
  // Saved by the forward (both or neither; tensor-core path): its output
  // [B,S,Hq,D] and row normalisers [B,Hq,S] (natural log).  Given, the dq
  // kernel takes Delta = dout . out and the log-sum-exp from them instead of
  // a first pass over the selected blocks.
  const void* out_in;
  const float* lse_in;
  int32_t* rev_off;        // scratch: [B,Hkv,nb+1] reverse-index offsets
  int32_t* rev;            // scratch: [B,Hkv,(Hq/Hkv)*nb*nsel] (local query head * nb + query block)
  float* dq;               // [B,S,Hq,D]
  float* dk;               // [B,S,Hkv,D]
  float* dv;               // [B,S,Hkv,D]
  int32_t* status;         // a selected id past its query block sets 2
  int B, S, Hq, Hkv, D, bs, nb, nsel;
  float scale;
  float inv_freq[64];
};
size_t bwd_rev_smem(int nb);
// Float32 storage: rotated float32 copies, reverse index, dq and dk/dv on the CUDA cores.
cudaError_t launch_backward(const BwdArgs& a, bool bf16, cudaStream_t st);
// Reverse index of the selection (key block -> selecting (query head, query block)).
cudaError_t launch_bwd_rev(const BwdArgs& a, cudaStream_t st);
// Bf16 storage, bs in {64,128}, D in {64,128}: reverse index, then dq and
// dk/dv on the tensor cores over qrot, krot (written by the summary kernel).
cudaError_t launch_backward_tc(const BwdArgs& a, cudaStream_t st);

}  // namespace mdr
