/*
 * mdr.h -- C ABI of libmdr: learned product-hash routed attention (forward)
 * on NVIDIA B200 (sm_100a).
 *
 * The method (pages cited by title and section):
 *   "Monodratic: a reproducible sparse attention mixer" (technical report
 *   summary; "Report" below) and "Monodratic Claims Learned Routing Can Make
 *   Sparse Causal Attention More Selective" ("Article" below).
 *
 *   After rotary position embedding, every source block of keys gets a
 *   product address from P codebooks and is written into a bounded causal
 *   posting list; every query block probes addresses, gathers the listed
 *   earlier blocks as candidates, reranks them and keeps R remote blocks,
 *   adds L local blocks, and runs ordinary causal softmax over the tokens of
 *   the selected blocks (Report, "Mixer"; Article, "Monodratic Turns Sparse
 *   Attention Into a Retrieval Decision").
 *
 * Conventions shared by every entry point
 *   - Every pointer argument named "device" points to GPU memory of the
 *     current device; "host" pointers point to CPU memory (pinned memory
 *     makes the copies asynchronous).  The caller owns every buffer; the
 *     library allocates nothing and keeps no state between calls, except
 *     mdr_route_noalloc, whose scratch is an array inside the library, and
 *     mdr_forward_host, which keeps two streams and nine events per device
 *     from its first call on (calls on one device run one at a time).
 *   - Layouts are C-contiguous.  q is [B,S,Hq,D]; k and v are [B,S,Hkv,D];
 *     out is [B,S,Hq,D]; all four have the element type cfg->dtype.
 *     Query head hq reads KV head hq / (Hq/Hkv).
 *   - codebooks are float32 [P,K,D/P]: P codebooks of K codewords, one per
 *     contiguous subspace of D/P coordinates.  They are used as given (the
 *     library does not renormalise them).
 *   - "stream" is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Device work is enqueued on it and the call returns without
 *     synchronising, except mdr_forward_host and mdr_read_device_status.
 *   - Argument checks run on the host before anything is enqueued; a failed
 *     check returns its status and enqueues nothing.  They touch no GPU, so
 *     they also work on a machine without one.
 *   - Kernels that wait on asynchronous copies or tensor-core work bound every
 *     wait; a wait that runs out sets a nonzero code in the device status
 *     word (the first 4 bytes of the workspace) and the kernel returns.  Read
 *     it with mdr_read_device_status after the call.
 */
#ifndef MDR_H_
#define MDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MDR_ABI_VERSION 1

typedef enum mdr_status {
  MDR_OK = 0,
  MDR_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, inconsistent shape */
  MDR_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement */
  MDR_ERR_WORKSPACE = 3,     /* workspace missing, too small or not 256-byte aligned */
  MDR_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  MDR_ERR_DEVICE = 5         /* the device status word reports a failed check */
} mdr_status;

typedef enum mdr_dtype { MDR_F32 = 0, MDR_BF16 = 1 } mdr_dtype;

/* Shapes and routing parameters of one call.
 *   B, S, Hq, Hkv, D : batch, tokens, query heads, KV heads, head dimension.
 *   block            : tokens per block (bs); S % block == 0, nb = S / block.
 *   P, K             : P codebooks of K codewords; A = K^P addresses.
 *   cap              : capacity of each posting list (blocks).
 *   probes           : codewords probed per subspace (p); p^P addresses probed.
 *   R, L             : remote blocks kept, local blocks added (L >= 1).
 *   rope_base        : rotary base (10000 in the pages' tiny case).
 *   scale            : softmax scale; 0 means 1/sqrt(D).
 *   dtype            : mdr_dtype of q, k, v, out.
 * Supported: D in {32,64,128}; block in {16,32,64,128}; 1 <= P <= 4 with
 * D % P == 0 and (D/P) % 4 == 0; 1 <= K <= 128; A <= 16384; 1 <= cap <= 1024;
 * 1 <= probes <= K with probes^P <= 64 and probes^P * cap <= 4096;
 * 0 <= R <= 32; 1 <= L <= 32; S/block <= 32768.  MDR_BF16 additionally needs block in {64,128}
 * and D in {64,128} (the tensor-core attention tiles).                      */
typedef struct mdr_config {
  int32_t B, S, Hq, Hkv, D, block;
  int32_t P, K, cap, probes, R, L;
  float rope_base;
  float scale;
  int32_t dtype;
} mdr_config;

/* The index of every (sequence, KV head); all device pointers, all required.
 *   kbar     float32 [B,Hkv,nb,D]  mean rotated key of each block.
 *   addr     int32   [B,Hkv,nb]    product address of each block, in [0, A).
 *   lists    int32   [B,Hkv,A,cap] posting lists: the first cap blocks (in
 *                                  ascending block order) hashed to each
 *                                  address, -1 padded.
 *   load     int32   [B,Hkv,A]     blocks hashed to each address (uncapped:
 *                                  the assigned load of Report, Capacity).
 *   overflow int32   [B,Hkv]       blocks not stored: sum of max(0, load-cap).
 *   maxload  int32   [B,Hkv]       largest load.                              */
typedef struct mdr_index {
  float* kbar;
  int32_t* addr;
  int32_t* lists;
  int32_t* load;
  int32_t* overflow;
  int32_t* maxload;
} mdr_index;

/* Route outputs; device pointers.  sel is required, the others may be NULL.
 *   sel    int32   [B,Hq,nb,R+L] selected blocks of each query block: the
 *                                remote blocks in ascending order, -1 where
 *                                fewer than R candidates exist, then the
 *                                local blocks j-L+1..j (-1 where negative).
 *   qbar   float32 [B,Hq,nb,D]   mean rotated query of each block.
 *   qcodes int32   [B,Hq,nb,P,probes] probed codewords per subspace, best
 *                                first.
 *   ncand  int32   [B,Hq,nb]     eligible candidates found in the probed
 *                                lists (at most probes^P * cap).            */
typedef struct mdr_route_out {
  int32_t* sel;
  float* qbar;
  int32_t* qcodes;
  int32_t* ncand;
} mdr_route_out;

/* Library and ABI version; MDR_ABI_VERSION of the build. */
int32_t mdr_abi_version(void);

/* Static text for a status code. */
const char* mdr_status_string(mdr_status s);

/* Check a configuration (the rules listed at mdr_config). */
mdr_status mdr_check_config(const mdr_config* cfg);

/* Device workspace the device entry points need, in bytes (host only). */
mdr_status mdr_workspace_bytes(const mdr_config* cfg, size_t* bytes);

/* Index: rotate the keys, average each block, give each block a product
 * address made of one codeword choice per subspace, and write the blocks
 * into bounded causal posting lists, counting overflow (Article, "Monodratic
 * Turns Sparse Attention Into a Retrieval Decision"; Report, sections Mixer
 * and Capacity).  k: device [B,S,Hkv,D]; codebooks: device.                */
mdr_status mdr_build_index(const mdr_config* cfg, const void* k,
                           const float* codebooks, const mdr_index* idx,
                           void* ws, size_t ws_bytes, void* stream);

/* Route: rotate the queries, average each block, probe the p best codewords
 * per subspace, gather the listed blocks i <= j-L as candidates in fixed
 * slots, rerank by <qbar_j, kbar_i> (float32), keep the R best (ties to the
 * lower block id) and add the L local blocks (Article, "Monodratic Turns
 * Sparse Attention Into a Retrieval Decision": probe, candidates, rerank, a
 * fixed count of remote blocks, local blocks always added).
 * q: device [B,S,Hq,D]; idx as filled by mdr_build_index (kbar, lists, load
 * are read).                                                                 */
mdr_status mdr_route(const mdr_config* cfg, const void* q,
                     const float* codebooks, const mdr_index* idx,
                     const mdr_route_out* rt, void* ws, size_t ws_bytes,
                     void* stream);

/* Attend: for token t of block j, causal softmax of scale*<q'_t, k'_s> over
 * every token s <= t of the blocks in sel[j], applied to v_s; q', k' are the
 * rotated queries and keys; exact softmax over the selected tokens, the
 * values used as they are (Report, section Mixer).  sel: device int32 [B,Hq,nb,R+L]; any valid block id in
 * [0, j] may appear, -1 entries are skipped, ids must not repeat within a
 * row; an id outside [0, j] is skipped and sets status 2.  A query block
 * left with no valid block gets a zero output.  out: device [B,S,Hq,D].
 * bf16 runs on the tensor cores (tcgen05, TMEM accumulators, TMA loads);
 * float32 runs on the CUDA cores in float32.                                             */
mdr_status mdr_attend(const mdr_config* cfg, const void* q, const void* k,
                      const void* v, const int32_t* sel, void* out, void* ws,
                      size_t ws_bytes, void* stream);

/* The whole forward, index -> route -> attend, with the rotation and the
 * summaries of both sides computed once.                                    */
mdr_status mdr_forward(const mdr_config* cfg, const void* q, const void* k,
                       const void* v, const float* codebooks,
                       const mdr_index* idx, const mdr_route_out* rt,
                       void* out, void* ws, size_t ws_bytes, void* stream);

/* mdr_attend / mdr_forward for training: the same output, and besides it
 * each row's softmax normaliser, lse[b,hq,t] = log of the sum over the
 * row's visible keys s of exp(scale*<q'_t, k'_s>) (natural log; -inf for a
 * query block with no valid selected block), which mdr_attend_backward_saved
 * reuses.  lse: device float32 [B,Hq,S], required.                          */
mdr_status mdr_attend_train(const mdr_config* cfg, const void* q, const void* k,
                            const void* v, const int32_t* sel, void* out,
                            float* lse, void* ws, size_t ws_bytes, void* stream);
mdr_status mdr_forward_train(const mdr_config* cfg, const void* q, const void* k,
                             const void* v, const float* codebooks,
                             const mdr_index* idx, const mdr_route_out* rt,
                             void* out, float* lse, void* ws, size_t ws_bytes,
                             void* stream);

/* mdr_forward that also records CUDA events at the kernel boundaries, for
 * timing each kernel on the stream it runs on.  events: host array of
 * n_events cudaEvent_t (as void*), each NULL to skip; events[0] before the
 * first kernel, events[1] after the summary kernel, events[2] after the
 * list kernel, events[3] after the route kernel, events[4] after the
 * attention kernel.  Same work and outputs as mdr_forward.                   */
mdr_status mdr_forward_profiled(const mdr_config* cfg, const void* q,
                                const void* k, const void* v,
                                const float* codebooks, const mdr_index* idx,
                                const mdr_route_out* rt, void* out, void* ws,
                                size_t ws_bytes, void* stream,
                                void* const* events, int32_t n_events);

/* Device workspace mdr_forward_host needs, in bytes (host only).           */
mdr_status mdr_host_workspace_bytes(const mdr_config* cfg, size_t* bytes);

/* The forward from host buffers: copies q, k, v, codebooks to the device
 * workspace, runs the forward there, copies out, sel, overflow and maxload
 * back, and synchronises before returning.  The forward is causal (block j's
 * output needs the inputs of blocks <= j only), so it runs in up to four
 * chunks of query blocks: a chunk's inputs are copied in on one internal
 * stream, its blocks summarised, appended to the posting lists, routed and
 * attended on `stream`, and its output copied out on another internal
 * stream while the next chunk's inputs come in.  The results are
 * bit-identical to mdr_forward.  The copies overlap only from pinned host
 * memory.  q, k, v, codebooks, out: host; sel_host [B,Hq,nb,R+L],
 * overflow_host and maxload_host [B,Hkv]: host int32 (each may be NULL to
 * skip its copy).  dev_ws: device, at least mdr_host_workspace_bytes.  Work
 * enqueued on `stream` before the call comes first.                         */
mdr_status mdr_forward_host(const mdr_config* cfg, const void* q_host,
                            const void* k_host, const void* v_host,
                            const float* codebooks_host, void* out_host,
                            int32_t* sel_host, int32_t* overflow_host,
                            int32_t* maxload_host, void* dev_ws,
                            size_t dev_ws_bytes, void* stream);

/* The route step without any workspace, for callers that can neither pass
 * a workspace nor call cudaMalloc (a serving loop whose device memory is all
 * reserved by its own pool, a plugin interface that hands an operator only
 * its inputs and outputs).  The pages have no counterpart: this exists only
 * for such callers.  Same inputs and outputs as mdr_route (sel required,
 * ncand may be NULL; the query summaries and probe codes are not returned).
 * Its scratch (query block means and probe codewords) lives in a 32 MiB
 * array inside the library, held on every GPU that loads it until exit; it
 * needs B*Hq*nb*(4*D + 4*P*probes) bytes (each part rounded up to 256) and
 * larger calls return MDR_ERR_WORKSPACE before anything is enqueued.  The
 * first call on each device looks up the array's device address with that
 * device current; it returns MDR_ERR_INVALID_ARG if the stream is capturing
 * then, so make it before any stream capture.  Calls share the array and a
 * device status word, so calls that overlap on the GPU race; the word is
 * cleared at the start of each call and the array needs no clearing.  If a
 * bounded wait of the summary step runs out on the device, every sel row is
 * written as -1 and ncand as -1: sel[b,hq,j,R+L-1] (the query block itself
 * in a normal route) is then -1, which is how the caller detects it after
 * synchronising.  Allocates nothing.                                        */
mdr_status mdr_route_noalloc(const mdr_config* cfg, const void* q,
                             const float* codebooks, const mdr_index* idx,
                             int32_t* sel, int32_t* ncand, void* stream);

/* ------------------------------------------------ controls and diagnostics
 * The controls the pages run beside the learned route (Report, section
 * Learned sparse route; Article, "Why Learned Product-Hash Routing Matters
 * Now"): the local-only control is any call with R = 0; the untrained-router
 * control is any call with random unit codebooks; the forced-target run and
 * the target-block hit rate (Report, section Evidence) are these two calls. */

/* mdr_route with a forced target block per route: the labelled target is put
 * into the selected set under the same budget of R remote blocks.  force:
 * device int32 [B,Hq,nb] (required).  Where 0 <= force[b,hq,j] <= j-L and
 * R > 0, the remote part of sel[b,hq,j] is the forced block plus the R-1
 * best other candidates (so the target replaces the weakest choice when the
 * route missed it and changes nothing when it found it), in ascending order
 * like every sel row; any other value (-1 for no target, a local block, a
 * later block) leaves the route as mdr_route computes it.  ncand counts the
 * eligible candidates the probes found, as in mdr_route.  Other arguments
 * and outputs as mdr_route.                                                 */
mdr_status mdr_route_forced(const mdr_config* cfg, const void* q,
                            const float* codebooks, const mdr_index* idx,
                            const int32_t* force, const mdr_route_out* rt,
                            void* ws, size_t ws_bytes, void* stream);

/* Target-block hits: for every route (b, hq, j) with target[b,hq,j] >= 0,
 * whether that block id appears anywhere in sel[b,hq,j] (remote or local
 * part).  sel: device int32 [B,Hq,nb,R+L] as written by a route call;
 * target: device int32 [B,Hq,nb], -1 = no target; hit: device int32
 * [B,Hq,nb] or NULL: 1 hit, 0 miss, -1 no target; counts: device int32 [2],
 * written (not accumulated): counts[0] = routes with a target, counts[1] =
 * hits.  The hit rate is counts[1] / counts[0].  Needs no workspace.        */
mdr_status mdr_target_hits(const mdr_config* cfg, const int32_t* sel,
                           const int32_t* target, int32_t* hit,
                           int32_t* counts, void* stream);

/* ------------------------------------------------------------- decoding
 * One token at a time with an incremental index.  The pages leave decoding
 * open and ask that a deployed decoder update its routing structures as
 * tokens arrive while keeping causality (Article, on what a deployed decoder
 * must do; bounded lists keep each update O(1)).  Here a block enters the
 * index when its last token arrives -- summary, address and list append as
 * in mdr_build_index, so a decoder and a prefill of the same prefix hold the
 * same lists -- and the new token t of block j = t / block is routed by its
 * own rotated query (a block of one token): candidates i <= j-L from the
 * probed lists, top R by <q'_t, kbar_i>, locals j-L+1..j, then causal
 * softmax over the selected tokens s <= t.
 *
 * Decode state: everything a decoder keeps between tokens; device memory,
 * caller-owned, sized by cfg (S = capacity in tokens, nb = S / block).
 *   krot  cfg->dtype [B,S,Hkv,D]  rotated keys of the tokens seen so far.
 *   v     cfg->dtype [B,S,Hkv,D]  their values.
 *   ksum  float32    [B,Hkv,D]    float32 sum of the rotated keys of the
 *                                 current, incomplete block (its summary is
 *                                 taken from these, not from the rounded
 *                                 cache).
 *   idx   mdr_index of the completed blocks (kbar and addr rows of blocks
 *         not yet complete are undefined).                                */
typedef struct mdr_decode_state {
  void* krot;
  void* v;
  float* ksum;
  mdr_index idx;
} mdr_decode_state;

/* Device workspace mdr_decode_prefill and mdr_decode_step need, in bytes
 * (host only); the first 4 bytes are the device status word.              */
mdr_status mdr_decode_workspace_bytes(const mdr_config* cfg, size_t* bytes);

/* Empty state (no token seen): lists -1, load, overflow, maxload and ksum 0. */
mdr_status mdr_decode_reset(const mdr_config* cfg, const mdr_decode_state* st,
                            void* stream);

/* State after the first S0 tokens (0 <= S0 <= cfg->S, S0 % block == 0):
 * rotates their keys into st->krot, copies their values into st->v and
 * builds the index of their S0/block blocks with the prefill kernels; the
 * rest of the state is reset.  k, v: device [B,S0,Hkv,D]; codebooks: device. */
mdr_status mdr_decode_prefill(const mdr_config* cfg, int32_t S0, const void* k,
                              const void* v, const float* codebooks,
                              const mdr_decode_state* st, void* ws,
                              size_t ws_bytes, void* stream);

/* One token at position t (0 <= t < cfg->S) of every sequence; the state
 * must hold tokens 0..t-1 (from mdr_decode_prefill and earlier steps; the
 * library cannot check this).  Stores the token's rotated key and value,
 * completes block t/block when t is its last token, routes the token and
 * writes its attention output.  q_t: device [B,Hq,D]; k_t, v_t: device
 * [B,Hkv,D]; out_t: device [B,Hq,D] (all cfg->dtype); sel_t: device int32
 * [B,Hq,R+L] (remote ids ascending, -1 pads, then the locals; required);
 * ncand_t: device int32 [B,Hq] eligible candidates found (may be NULL).     */
mdr_status mdr_decode_step(const mdr_config* cfg, int32_t t, const void* q_t,
                           const void* k_t, const void* v_t,
                           const float* codebooks, const mdr_decode_state* st,
                           void* out_t, int32_t* sel_t, int32_t* ncand_t,
                           void* ws, size_t ws_bytes, void* stream);

/* Synchronise the stream and copy the device status word (first 4 bytes of
 * ws) to *code (0 = no device-side failure).  Returns MDR_ERR_DEVICE when the
 * word is nonzero.                                                           */
mdr_status mdr_read_device_status(const void* ws, int32_t* code, void* stream);

/* ------------------------------------------------------------- backward
 * Gradients of the attention output with the route held fixed.  The pages
 * note that hard top-k choices give no ordinary gradient through the chosen
 * index and leave surrogates to the trainer (Article, "The 99.35 Percent
 * Result Does Not Establish Language Quality"); this is the gradient of
 * mdr_attend's output with respect to q, k and v for a given sel:
 *   for token t of block j and every selected token s <= t,
 *   P = softmax(scale*<q'_t, k'_s>), dv_s += P dout_t,
 *   dS = P (<dout_t, v_s> - <dout_t, out_t>),
 *   dq'_t += scale dS k'_s, dk'_s += scale dS q'_t,
 *   dq = R(t)^T dq', dk = R(s)^T dk' (the transpose of the rotation);
 * key and value gradients of a KV head add over its query heads; a query
 * block with no valid selected block gets zero gradients.  Nothing reaches
 * the codebooks or the summaries.
 * q, k, v: device [B,S,H,D] in cfg->dtype (not rotated: the inputs of
 * mdr_forward); sel: device int32 [B,Hq,nb,R+L] as written by a route call;
 * dout: device [B,S,Hq,D] in cfg->dtype; dq [B,S,Hq,D], dk and dv
 * [B,S,Hkv,D]: device float32, written (not accumulated).  MDR_BF16: the
 * four products run on the tensor cores (tcgen05) with bfloat16 operands --
 * the rotated q', k' the forward uses, and the weights P, dS -- accumulated
 * in float32 (q, k, v, dout, dq, dk, dv 16-byte aligned, else
 * MDR_ERR_INVALID_ARG); MDR_F32: float32 on the CUDA cores.  Either way the
 * sums run in a fixed order (deterministic).  ws: device, 256-byte aligned,
 * at least mdr_backward_workspace_bytes; its first word is the device
 * status (2: a selected id later than its query block, skipped), read with
 * mdr_read_device_status.  Supported up to 29,000 blocks per sequence
 * (S/block; the reverse index of a (sequence, KV head) lives in shared
 * memory), else MDR_ERR_UNSUPPORTED before anything is enqueued.            */
mdr_status mdr_backward_workspace_bytes(const mdr_config* cfg, size_t* bytes);
mdr_status mdr_attend_backward(const mdr_config* cfg, const void* q, const void* k,
                               const void* v, const int32_t* sel, const void* dout,
                               float* dq, float* dk, float* dv, void* ws,
                               size_t ws_bytes, void* stream);

/* mdr_attend_backward with the forward's output and row normalisers saved
 * by mdr_attend_train / mdr_forward_train (out: device [B,S,Hq,D] in
 * cfg->dtype, 16-byte aligned for MDR_BF16; lse: device float32 [B,Hq,S];
 * both required, both from the same sel).  MDR_BF16 takes
 * Delta_t = <dout_t, out_t> and the normalisers from them and so skips the
 * first of its two passes over the selected blocks; MDR_F32 recomputes them
 * as mdr_attend_backward does.  Same outputs, workspace and status.         */
mdr_status mdr_attend_backward_saved(const mdr_config* cfg, const void* q,
                                     const void* k, const void* v,
                                     const int32_t* sel, const void* out,
                                     const float* lse, const void* dout,
                                     float* dq, float* dk, float* dv, void* ws,
                                     size_t ws_bytes, void* stream);

/* ------------------------------------------------- codebook calibration
 * Spherical codebook calibration (Report, section Capacity and Figure 3:
 * codebooks calibrated on a training split remove held-out overflow and
 * lower the maximum assigned load).  The pages give the method's name, not
 * its steps; this is spherical k-means per subspace, started from the
 * given codebooks.  Each round:
 *   assign  record x goes to the codeword of largest <x_s, C[s,k]> in each
 *           subspace s (float32, lower index on equal scores: the address
 *           code of mdr_build_index);
 *   update  C[s,k] = the normalised sum of x_s/|x_s| over its members;
 *           records whose x_s has no nonzero coordinate are not members; a
 *           codeword with no member or a zero sum keeps its value.
 * Sums run in a fixed order (float32), so a call is deterministic.
 *
 * records: device float32 [N,D], 16-byte aligned -- e.g. the block
 *   summaries of a training split (mdr_index.kbar and mdr_route_out.qbar are
 *   such arrays, [B,H,nb,D] = [N,D] with N = B*H*nb).
 * codebooks_in, codebooks_out: device float32 [P,K,D/P], 16-byte aligned;
 *   equal (in place) or disjoint.
 * rounds: >= 0; 0 copies codebooks_in to codebooks_out.
 * counts: device int32 [P,K] or NULL: members of each codeword in the last
 *   round.  assign: device int32 [N,P] or NULL: each record's codeword in
 *   the last round (the assignment to the codebooks that round started
 *   from).
 * ws: device, 256-byte aligned, at least mdr_calibrate_workspace_bytes.
 * Supported: D in {32,64,128}, 1 <= P <= 4, D/P a multiple of 4 and >= 8,
 * 1 <= K <= 128, 1 <= N <= 2^31/P (else MDR_ERR_UNSUPPORTED or
 * MDR_ERR_INVALID_ARG, checked on the host before anything is enqueued).  */
mdr_status mdr_calibrate_workspace_bytes(int64_t N, int32_t D, int32_t P, int32_t K,
                                         size_t* bytes);
mdr_status mdr_calibrate_codebooks(const float* records, int64_t N, int32_t D,
                                   int32_t P, int32_t K, const float* codebooks_in,
                                   float* codebooks_out, int32_t rounds,
                                   int32_t* counts, int32_t* assign, void* ws,
                                   size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MDR_H_ */
