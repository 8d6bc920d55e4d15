"""CPU oracle of the learned product-hash routed-attention forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module.  It shares no code with the CUDA
library and imports nothing from it.

It is written to be read against the two pages that describe the method:

  Report  = "Monodratic: a reproducible sparse attention mixer" (D. Todorov,
            technical report summary), sections Mixer, Learned sparse route,
            Capacity, Finite-range scaling, Evidence, Limits, Figures 1-4.
  Article = "Monodratic Claims Learned Routing Can Make Sparse Causal Attention
            More Selective" (remio.ai), section "Monodratic Turns Sparse
            Attention Into a Retrieval Decision" unless stated.

The forward is index -> route -> attend:
  1. rotary embedding of queries and keys (Report, Mixer; Article);
  2. per-block summaries of the rotated queries and keys;
  3. a product address per source block: one codeword choice per subspace,
     combined (Article; Report, Capacity, for the spherical codebooks);
  4. bounded causal posting lists, overflow counted (Report, Mixer; Report,
     Capacity and Evidence: overflow events, maximum assigned load);
  5. probe -> candidates in fixed slots -> rerank -> R remote blocks, plus L
     local blocks added separately (Article; Report, Mixer; Report,
     Finite-range scaling, for the fixed candidate slots);
  6. exact causal softmax over the tokens of the selected blocks, with their
     own values (Report, Mixer; Article).
And the independent dense selected-mask form of step 6 (Report, Evidence,
the selected-mask oracle row; Article, "Why Learned Product-Hash Routing
Matters Now").  Beyond the forward (sections 7-9 and the route's options):
  7. decode: one token at a time with an incremental index;
  -  controls: a forced target block per route (route_row's force) and the
     target-block hit count (target_hits);
  8. codebook calibration: spherical k-means per subspace;
  9. backward: gradients of the attention output with the route held fixed.

Precision.  Every value is computed in float64 from the stored inputs.  Two
readings fix what the pages leave open (both recorded with the others in the
design notes):
  * the rotary angle is the float32 product fp32(t) * fp32(base**(-2i/D)),
    the way a float32 PyTorch rotary table is built; its cosine and sine are
    then taken in float64;
  * a routing decision (an argmax, a top-p, a top-R) is taken on the deciding
    quantities rounded to float32, the precision the routing kernels decide
    in.  Equal float32 scores go to the lower index.  ``margin`` outputs give
    the float32 gap at each decision boundary so callers can tell a near tie.
Attention outputs stay in float64.
"""
from __future__ import annotations

import itertools
from dataclasses import dataclass, field

import numpy as np

TIE_REL = 1e-6   # a decision whose float32 margin is below 1e-6*max(1,|s|) is a near tie


def f32(x):
    """Round to float32 and return as float64 (the values a float32 kernel holds)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------- 1. rotary
def rope_inv_freq(D: int, base: float) -> np.ndarray:
    """omega_i = base**(-2i/D), i < D/2, rounded to float32."""
    i = np.arange(D // 2, dtype=np.float64)
    return np.array([base ** (-2.0 * ii / D) for ii in i]).astype(np.float32)


def rope_angles(S: int, D: int, base: float) -> np.ndarray:
    """Angle of pair i at position t: the float32 product fp32(t) * omega_i. [S, D/2]"""
    t = np.arange(S, dtype=np.float32)
    return (t[:, None] * rope_inv_freq(D, base)[None, :]).astype(np.float32)


def rope(x: np.ndarray, base: float) -> np.ndarray:
    """Rotary embedding of x [B,S,H,D] at absolute positions 0..S-1.

    Rotate-half pairing: coordinate i is paired with i + D/2 and the pair is
    rotated by the angle of position t and frequency i.  Applied to queries and
    keys, never to values (Report, Mixer: routing follows the rotation).
    """
    B, S, H, D = x.shape
    th = rope_angles(S, D, base).astype(np.float64)
    c = np.cos(th)[None, :, None, :]
    s = np.sin(th)[None, :, None, :]
    x1 = x[..., : D // 2]
    x2 = x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ------------------------------------------------------------- 2. summaries
def block_means(xr: np.ndarray, bs: int) -> np.ndarray:
    """Mean of the rotated vectors over each block of bs tokens.

    [B,S,H,D] -> [B,H,nb,D].  Source blocks and query blocks are both
    summarised this way (Article: addresses are given to source blocks; the
    query of a block is its mean rotated query).
    """
    B, S, H, D = xr.shape
    nb = S // bs
    return xr.reshape(B, nb, bs, H, D).mean(axis=2).transpose(0, 2, 1, 3)


# ------------------------------------------------------------------ 3. codes
def codeword_scores(xbar: np.ndarray, codebooks: np.ndarray) -> np.ndarray:
    """<xbar_s, C[s,k]> for every subspace s and codeword k, rounded to float32.

    xbar [..., D] is split into P contiguous subvectors of D/P.  The summary is
    not normalised: dividing by a positive norm does not change which codeword
    wins.  -> [..., P, K]
    """
    P, K, d = codebooks.shape
    sub = f32(xbar).reshape(*xbar.shape[:-1], P, d)
    return f32(np.einsum("...pd,pkd->...pk", sub, codebooks.astype(np.float64)))


def assign_codes(kbar: np.ndarray, codebooks: np.ndarray):
    """Product address of each source block.

    Per subspace the code is the codeword of largest score (lowest index on
    equal scores); the address is sum_s code_s * K**(P-1-s), the first
    subspace most significant.  Returns (addr [...], codes [..., P],
    margin [..., P] = best - second best score).
    """
    P, K, _ = codebooks.shape
    sc = codeword_scores(kbar, codebooks)
    codes = np.argmax(sc, axis=-1)                   # first maximum -> lowest index
    srt = -np.sort(-sc, axis=-1)
    margin = srt[..., 0] - srt[..., 1] if K > 1 else np.full(sc.shape[:-1], np.inf)
    weights = K ** np.arange(P - 1, -1, -1)
    addr = (codes * weights).sum(axis=-1)
    return addr.astype(np.int64), codes.astype(np.int64), margin


def code_scale(xbar: np.ndarray, codebooks: np.ndarray) -> np.ndarray:
    """Largest |codeword score| of each subspace: the |s| that sets the
    near-tie threshold of a code or probe decision.  -> [..., P]"""
    return np.abs(codeword_scores(xbar, codebooks)).max(axis=-1)


def probe_codes(qbar: np.ndarray, codebooks: np.ndarray, p: int):
    """The p best codewords per subspace for each query block.

    Ordered by score, highest first, lower index first on equal scores.
    Returns (codes [..., P, p], margin [..., P] = gap between ranks p and p+1).
    """
    P, K, _ = codebooks.shape
    sc = codeword_scores(qbar, codebooks)
    order = np.argsort(-sc, axis=-1, kind="stable")
    codes = order[..., :p]
    srt = np.take_along_axis(sc, order, axis=-1)
    margin = srt[..., p - 1] - srt[..., p] if p < K else np.full(sc.shape[:-1], np.inf)
    return codes.astype(np.int64), margin


def probe_addresses(codes_row: np.ndarray, K: int) -> np.ndarray:
    """Addresses probed by one query block: the product of its per-subspace
    codeword choices, enumerated with the first subspace's rank slowest.
    codes_row [P, p] -> [p**P]."""
    P, p = codes_row.shape
    weights = K ** np.arange(P - 1, -1, -1)
    out = []
    for ranks in itertools.product(range(p), repeat=P):
        out.append(sum(int(codes_row[s, r]) * int(weights[s]) for s, r in enumerate(ranks)))
    return np.array(out, dtype=np.int64)


# ------------------------------------------------------------ 4. posting lists
def build_lists(addr_row: np.ndarray, A: int, cap: int):
    """Bounded causal posting lists of one (sequence, KV head).

    Blocks are inserted in ascending block order; a block is stored if its
    address's list holds fewer than cap blocks, otherwise it is an overflow
    event.  Whether block i is stored depends only on blocks before it, so no
    later block can change what an earlier query sees.  load counts every block
    hashed to the address (the "assigned load", which may exceed capacity).
    Returns lists [A, cap] (-1 padded, ascending), load [A], overflow, maxload.
    """
    lists = np.full((A, cap), -1, dtype=np.int64)
    load = np.zeros(A, dtype=np.int64)
    for i, a in enumerate(addr_row):
        if load[a] < cap:
            lists[a, load[a]] = i
        load[a] += 1
    overflow = int(np.maximum(load - cap, 0).sum())
    return lists, load, overflow, int(load.max()) if A else 0


# ------------------------------------------------------------------- 5. route
@dataclass
class RouteRow:
    sel: np.ndarray          # [R+L]: remote ids ascending, -1 pads, then locals
    slots: np.ndarray        # [p**P, cap] fixed candidate slots (-1 = empty)
    cand: np.ndarray         # eligible candidate ids
    scores: np.ndarray       # float32 scores of the ranked pool (the candidates, less a forced id)
    margin: float            # score gap between the last kept rank and the next (inf if none)
    scale: float             # largest |score| in the pool (0 if empty): the near-tie reference


def candidate_slots(lists: np.ndarray, probe_addrs: np.ndarray, j: int, L: int) -> np.ndarray:
    """The fixed candidate slots of query block j: one row of cap slots per
    probed address, holding the listed blocks that are remote-eligible
    (i <= j - L); every other slot is -1.  Always p**P x cap."""
    slots = lists[probe_addrs].copy()
    slots[(slots < 0) | (slots > j - L)] = -1
    return slots


def route_row(qbar_j: np.ndarray, kbar_h: np.ndarray, probe_addrs: np.ndarray,
              lists: np.ndarray, j: int, R: int, L: int, force: int = -1) -> RouteRow:
    """Route one query block: probe -> candidates -> rerank -> top R, plus the
    L local blocks j-L+1..j (Article, section "Monodratic Turns Sparse
    Attention Into a Retrieval Decision": the query probes addresses, gets
    candidates, reranks them and keeps a fixed count of remote blocks; local
    blocks are always added).

    Rerank score of candidate i is <qbar_j, kbar_i> over the full head
    dimension, rounded to float32; top R by score, lower id on equal scores.
    The chosen remote ids are stored in ascending order.

    ``force`` is the forced-target diagnostic (Article, "Why Learned
    Product-Hash Routing Matters Now": the labelled target block is put into
    the selected set under the same attention budget).  Reading: when
    0 <= force <= j - L and R > 0, the remote set is the forced block plus
    the R - 1 best other candidates, so the target takes the place of the
    weakest choice when routing missed it and changes nothing when routing
    found it; any other value (no target, a local block, a later block)
    leaves the route as it is.
    """
    slots = candidate_slots(lists, probe_addrs, j, L)
    cand = slots[slots >= 0]
    forced = 0 <= force <= j - L and R > 0
    pool = cand[cand != force] if forced else cand
    keep = R - 1 if forced else R
    scores = f32(f32(kbar_h[pool]) @ f32(qbar_j)) if pool.size else np.zeros(0)
    order = np.lexsort((pool, -scores))
    top = pool[order[:keep]]
    if forced:
        top = np.concatenate([top, [force]])
    margin = np.inf
    if pool.size > keep and keep > 0:
        margin = float(scores[order[keep - 1]] - scores[order[keep]])
    remote = np.full(R, -1, dtype=np.int64)
    remote[: top.size] = np.sort(top)
    local = np.arange(j - L + 1, j + 1, dtype=np.int64)
    local[local < 0] = -1
    scale = float(np.abs(scores).max()) if scores.size else 0.0
    return RouteRow(np.concatenate([remote, local]), slots, cand, scores, margin, scale)


# ------------------------------------------------------------------ 6. attend
def selected_tokens(sel_row: np.ndarray, bs: int) -> np.ndarray:
    blocks = np.sort(sel_row[sel_row >= 0])
    return (blocks[:, None] * bs + np.arange(bs)[None, :]).ravel()


def attend(qr, kr, v, sel, bs: int, scale: float, rows=None) -> np.ndarray:
    """Exact causal softmax over the tokens of the selected blocks.

    For token t of query block j, head hq: the keys are every token s of every
    selected block with s <= t; weights softmax(scale * <q'_t, k'_s>) applied
    to v_s (Report, Mixer: exact causal softmax over the selected set, with the
    selected values, not a summary of them).  Query head hq reads KV
    head hq // (Hq/Hkv).  rows: optional list of (b, hq, j) to compute; the
    others stay NaN.  -> [B,S,Hq,D] float64.
    """
    B, S, Hq, D = qr.shape
    g = Hq // kr.shape[2]
    out = np.full((B, S, Hq, v.shape[3]), np.nan)
    nb = S // bs
    todo = rows if rows is not None else itertools.product(range(B), range(Hq), range(nb))
    for b, hq, j in todo:
        toks = selected_tokens(sel[b, hq, j], bs)
        qpos = np.arange(j * bs, (j + 1) * bs)
        Q = qr[b, qpos, hq]
        Kt = kr[b, toks, hq // g]
        Vt = v[b, toks, hq // g]
        s = (Q @ Kt.T) * scale
        s[toks[None, :] > qpos[:, None]] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        w = np.exp(s)
        out[b, qpos, hq] = (w @ Vt) / w.sum(axis=1, keepdims=True)
    return out


def softmax_lse(qr, kr, sel, bs: int, scale: float, rows=None) -> np.ndarray:
    """Log of the denominator of the softmax `attend` takes: for token t of
    query block j, head hq, log of the sum over every token s <= t of the
    selected blocks of exp(scale * <q'_t, k'_s>) (natural log; -inf when no
    block is selected).  The saved statistic a backward reuses (Report,
    Mixer: the exact causal softmax over the selected set).  rows: optional
    list of (b, hq, j); the others stay NaN.  -> [B,Hq,S] float64.
    """
    B, S, Hq, D = qr.shape
    g = Hq // kr.shape[2]
    out = np.full((B, Hq, S), np.nan)
    nb = S // bs
    todo = rows if rows is not None else itertools.product(range(B), range(Hq), range(nb))
    for b, hq, j in todo:
        toks = selected_tokens(sel[b, hq, j], bs)
        qpos = np.arange(j * bs, (j + 1) * bs)
        s = (qr[b, qpos, hq] @ kr[b, toks, hq // g].T) * scale
        s[toks[None, :] > qpos[:, None]] = -np.inf
        m = s.max(axis=1, initial=-np.inf)
        finite = np.isfinite(m)
        tot = np.where(finite[:, None], np.exp(s - np.where(finite, m, 0.0)[:, None]), 0.0).sum(axis=1)
        out[b, hq, qpos] = np.where(finite, m + np.log(np.where(finite, tot, 1.0)), -np.inf)
    return out


def selected_mask(sel_bh: np.ndarray, S: int, bs: int) -> np.ndarray:
    """Dense boolean [S, S] mask of one (sequence, head): M[t, s] is true when
    s's block is selected for t's block and s <= t."""
    nb = S // bs
    blk = np.zeros((nb, nb), dtype=bool)
    for j in range(nb):
        ids = sel_bh[j][sel_bh[j] >= 0]
        blk[j, ids] = True
    M = np.repeat(np.repeat(blk, bs, axis=0), bs, axis=1)
    return M & np.tril(np.ones((S, S), dtype=bool))


def attend_dense_mask(qr, kr, v, sel, bs: int, scale: float) -> np.ndarray:
    """The same attention as a dense masked softmax over all S keys, built
    independently of the gathered form (Report, Evidence: selected-mask
    oracle)."""
    B, S, Hq, D = qr.shape
    g = Hq // kr.shape[2]
    out = np.empty((B, S, Hq, v.shape[3]))
    for b in range(B):
        for hq in range(Hq):
            M = selected_mask(sel[b, hq], S, bs)
            s = (qr[b, :, hq] @ kr[b, :, hq // g].T) * scale
            s = np.where(M, s, -np.inf)
            s -= s.max(axis=1, keepdims=True)
            w = np.exp(s)
            out[b, :, hq] = (w @ v[b, :, hq // g]) / w.sum(axis=1, keepdims=True)
    return out


# ----------------------------------------------------------------- forward
@dataclass
class Params:
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int
    block: int
    P: int
    K: int
    cap: int
    probes: int
    R: int
    L: int
    rope_base: float = 10000.0
    scale: float = 0.0

    @property
    def nb(self):
        return self.S // self.block

    @property
    def A(self):
        return self.K ** self.P

    @property
    def softmax_scale(self):
        return self.scale if self.scale > 0 else 1.0 / np.sqrt(self.D)

    @classmethod
    def of(cls, w) -> "Params":
        return cls(**{f: getattr(w, f) for f in cls.__dataclass_fields__})


@dataclass
class Result:
    qr: np.ndarray
    kr: np.ndarray
    qbar: np.ndarray
    kbar: np.ndarray
    addr: np.ndarray
    codes: np.ndarray
    code_margin: np.ndarray
    qcodes: np.ndarray
    qcode_margin: np.ndarray
    lists: np.ndarray
    load: np.ndarray
    overflow: np.ndarray
    maxload: np.ndarray
    sel: np.ndarray
    sel_margin: np.ndarray
    ncand: np.ndarray
    out: np.ndarray | None = None
    slots: dict = field(default_factory=dict)
    sel_scale: np.ndarray | None = None     # [B,Hq,nb] largest |candidate score| per route
    v: np.ndarray | None = None             # the values, float64 (for re-running attention)


def build_index(kr, codebooks, p: Params, addr=None):
    """Index of every (sequence, KV head): summaries, addresses, lists.

    ``addr`` [B,Hkv,nb] (or None) replaces the computed addresses when the
    lists are built: where a code decision is a near tie either codeword is
    correct, so a check of what follows from another implementation's choice
    builds the lists from that choice.  codes and margins stay the computed
    ones."""
    kbar = block_means(kr, p.block)
    own_addr, codes, margin = assign_codes(kbar, codebooks)
    addr = own_addr if addr is None else np.asarray(addr, dtype=np.int64)
    B, H, nb = addr.shape
    lists = np.empty((B, H, p.A, p.cap), dtype=np.int64)
    load = np.empty((B, H, p.A), dtype=np.int64)
    overflow = np.empty((B, H), dtype=np.int64)
    maxload = np.empty((B, H), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            lists[b, h], load[b, h], overflow[b, h], maxload[b, h] = build_lists(addr[b, h], p.A, p.cap)
    return kbar, addr, codes, margin, lists, load, overflow, maxload


def route(qr, kbar, lists, codebooks, p: Params, keep_slots=False, force=None, qcodes=None):
    """Route every query block; ``force`` [B,Hq,nb] (or None) holds a forced
    target block per route, -1 for none (see route_row).  ``qcodes``
    [B,Hq,nb,P,p] (or None) replaces the computed probe codewords (a near-tie
    probe decision taken the other way); the returned qcodes and margins are
    the computed ones.  Returns (qbar, qcodes, qmargin, sel, sel_margin,
    ncand, slots, sel_scale)."""
    qbar = block_means(qr, p.block)
    own_qcodes, qmargin = probe_codes(qbar, codebooks, p.probes)
    use = own_qcodes if qcodes is None else np.asarray(qcodes, dtype=np.int64)
    B, Hq, nb = qbar.shape[:3]
    g = Hq // kbar.shape[1]
    sel = np.empty((B, Hq, nb, p.R + p.L), dtype=np.int64)
    sel_margin = np.empty((B, Hq, nb))
    sel_scale = np.empty((B, Hq, nb))
    ncand = np.empty((B, Hq, nb), dtype=np.int64)
    slots = {}
    for b in range(B):
        for hq in range(Hq):
            for j in range(nb):
                pa = probe_addresses(use[b, hq, j], p.K)
                row = route_row(qbar[b, hq, j], kbar[b, hq // g], pa,
                                lists[b, hq // g], j, p.R, p.L,
                                -1 if force is None else int(force[b, hq, j]))
                sel[b, hq, j] = row.sel
                sel_margin[b, hq, j] = row.margin
                sel_scale[b, hq, j] = row.scale
                ncand[b, hq, j] = row.cand.size
                if keep_slots:
                    slots[(b, hq, j)] = row.slots
    return qbar, own_qcodes, qmargin, sel, sel_margin, ncand, slots, sel_scale


def forward(q, k, v, codebooks, p: Params, *, attention=True, rows=None, keep_slots=False,
            force=None, addr=None, qcodes=None, sel=None) -> Result:
    """Index -> route -> attend for stored inputs q [B,S,Hq,D], k, v [B,S,Hkv,D];
    ``force`` as in route.

    Decision overrides (each None or an array of the decision's shape): where
    a decision is a near tie, either choice is correct, and the steps after it
    are checked against the oracle re-run with the other choice --
      addr   [B,Hkv,nb]      the lists are built from these addresses;
      qcodes [B,Hq,nb,P,p]   the routes probe these codewords;
      sel    [B,Hq,nb,R+L]   the attention runs over these selected blocks.
    The Result's addr, qcodes and sel are the ones used downstream (the
    overrides where given); the margins are those of the computed decisions,
    except sel_margin, which belongs to the routes run."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    qr = rope(q, p.rope_base)
    kr = rope(k, p.rope_base)
    kbar, own_addr, codes, cmargin, lists, load, overflow, maxload = build_index(kr, codebooks, p, addr)
    qbar, own_qcodes, qmargin, rsel, smargin, ncand, slots, sscale = route(
        qr, kbar, lists, codebooks, p, keep_slots, force, qcodes)
    use_addr = own_addr if addr is None else np.asarray(addr, dtype=np.int64)
    use_qcodes = own_qcodes if qcodes is None else np.asarray(qcodes, dtype=np.int64)
    use_sel = rsel if sel is None else np.asarray(sel, dtype=np.int64)
    out = attend(qr, kr, v, use_sel, p.block, p.softmax_scale, rows) if attention else None
    return Result(qr, kr, qbar, kbar, use_addr, codes, cmargin, use_qcodes, qmargin, lists, load,
                  overflow, maxload, use_sel, smargin, ncand, out, slots, sscale, v)


def target_hits(sel: np.ndarray, target: np.ndarray):
    """Target-block hit diagnostic (Report, Evidence: the target-block hit
    rate).  For every route with a target (target[b,hq,j] >= 0), whether that
    block is in the route's selected set (remote or local part); routes with
    no target (-1) are not counted.  Returns (hit [B,Hq,nb]: 1 hit, 0 miss,
    -1 no target; number of routes with a target; number of hits)."""
    B, Hq, nb = target.shape
    hit = np.full((B, Hq, nb), -1, dtype=np.int64)
    for b in range(B):
        for hq in range(Hq):
            for j in range(nb):
                t = int(target[b, hq, j])
                if t >= 0:
                    hit[b, hq, j] = 1 if t in set(int(x) for x in sel[b, hq, j]) else 0
    return hit, int((hit >= 0).sum()), int((hit == 1).sum())


def near_tie(margin, scale_ref) -> np.ndarray:
    """True where a float32 decision margin is below 1e-6*max(1,|s|)."""
    return np.asarray(margin) < TIE_REL * np.maximum(1.0, np.abs(scale_ref))


# ------------------------------------------------------------------ 7. decode
# Decoding one token at a time with an incremental index.  The pages ask that
# a deployed decoder update its routing structures as tokens arrive and keep
# causality ("Monodratic Claims Learned Routing Can Make Sparse Causal
# Attention More Selective", the section on what a deployed decoder must do;
# the bounded lists make the update O(1)).  Readings (listed with the others
# in the design notes):
#   * a block enters the index when its last token arrives: its summary is
#     the mean of its rotated keys, its address is assigned as in the batch
#     build, and it is appended to its list if the list holds fewer than cap
#     blocks -- exactly the batch build run one block at a time, so a decoder
#     and a prefill of the same prefix hold the same index;
#   * the new token t is routed by its own rotated query (a block of one
#     token), with eligibility i <= j - L and local blocks j-L+1..j taken
#     from its block j = t // bs; the current block is partly filled and the
#     causal mask keeps s <= t.


def rope_at(x: np.ndarray, t: int, base: float) -> np.ndarray:
    """Rotary embedding of vectors x [..., D] at the single position t (the
    same float32 angles as rope())."""
    D = x.shape[-1]
    th = (np.float32(t) * rope_inv_freq(D, base)).astype(np.float32).astype(np.float64)
    c, s = np.cos(th), np.sin(th)
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


@dataclass
class DecodeState:
    """Rotated keys and values seen so far and, per (sequence, KV head), the
    summaries, addresses and bounded lists of the completed blocks."""
    kr: np.ndarray          # [B, Smax, Hkv, D] rotated keys (positions < t)
    v: np.ndarray           # [B, Smax, Hkv, D]
    kbar: np.ndarray        # [B, Hkv, nbmax, D]
    addr: np.ndarray        # [B, Hkv, nbmax] (-1 until the block completes)
    lists: np.ndarray       # [B, Hkv, A, cap]
    load: np.ndarray        # [B, Hkv, A]
    t: int = 0              # tokens seen

    @property
    def overflow(self):
        cap = self.lists.shape[-1]
        return np.maximum(self.load - cap, 0).sum(axis=-1)

    @property
    def maxload(self):
        return self.load.max(axis=-1)


def decode_init(p: Params, B: int) -> DecodeState:
    """Empty state for sequences of up to p.S tokens."""
    return DecodeState(np.zeros((B, p.S, p.Hkv, p.D)), np.zeros((B, p.S, p.Hkv, p.D)),
                       np.zeros((B, p.Hkv, p.nb, p.D)), np.full((B, p.Hkv, p.nb), -1, dtype=np.int64),
                       np.full((B, p.Hkv, p.A, p.cap), -1, dtype=np.int64),
                       np.zeros((B, p.Hkv, p.A), dtype=np.int64))


def append_block(st: DecodeState, codebooks: np.ndarray, p: Params, j: int, addr=None):
    """Block j has all its tokens: summarise it, give it an address and append
    it to its list if that list holds fewer than cap blocks (load counts it in
    any case).  ``addr`` [B, Hkv] (or None) replaces the computed address (a
    near-tie code decision taken the other way).  Returns the computed
    (addr, codes, margin) of the block."""
    toks = st.kr[:, j * p.block:(j + 1) * p.block]                 # [B, bs, Hkv, D]
    st.kbar[:, :, j] = toks.mean(axis=1)
    own = assign_codes(st.kbar[:, :, j], codebooks)                  # [B, Hkv], ...
    addr = own[0] if addr is None else np.asarray(addr, dtype=np.int64)
    st.addr[:, :, j] = addr
    B, H = addr.shape
    for b in range(B):
        for h in range(H):
            a = addr[b, h]
            if st.load[b, h, a] < p.cap:
                st.lists[b, h, a, st.load[b, h, a]] = j
            st.load[b, h, a] += 1
    return own


@dataclass
class DecodeOut:
    out: np.ndarray          # [B, Hq, D] attention output of token t
    sel: np.ndarray          # [B, Hq, R+L]
    sel_margin: np.ndarray   # [B, Hq] top-R margin (float32 scores)
    qcodes: np.ndarray       # [B, Hq, P, p]
    qcode_margin: np.ndarray  # [B, Hq, P]
    ncand: np.ndarray        # [B, Hq]
    qcode_scale: np.ndarray  # [B, Hq, P] largest |codeword score| (reference for near ties)
    sel_scale: np.ndarray    # [B, Hq] largest |candidate score| (reference for near ties)
    # the block completed by this token (None if none): its computed address,
    # codes, code margins [B, Hkv, P] and largest |codeword score| [B, Hkv, P]
    key_addr: np.ndarray | None = None
    key_codes: np.ndarray | None = None
    key_margin: np.ndarray | None = None
    key_scale: np.ndarray | None = None


def decode_step(st: DecodeState, q_t, k_t, v_t, codebooks, p: Params, *, addr=None, sel=None) -> DecodeOut:
    """Token t = st.t of every sequence: store its rotated key and value,
    complete a block if t is its last token, then route the token by its
    rotated query and attend over the selected tokens s <= t.
    q_t [B, Hq, D], k_t and v_t [B, Hkv, D] (stored inputs).

    Decision overrides (near-tie decisions taken the other way, so that what
    follows is checked against that choice): ``addr`` [B, Hkv] is the address
    of the block this token completes; ``sel`` [B, Hq, R+L] is the selection
    the attention runs over.  The returned sel, margins and key decision are
    the computed ones; out is the attention over the selection used."""
    t = st.t
    q_t, k_t, v_t = (np.asarray(x, dtype=np.float64) for x in (q_t, k_t, v_t))
    st.kr[:, t] = rope_at(k_t, t, p.rope_base)
    st.v[:, t] = v_t
    key = (None, None, None, None)
    if (t + 1) % p.block == 0:
        j_done = t // p.block
        ka, kc, km = append_block(st, codebooks, p, j_done, addr)
        key = (ka, kc, km, code_scale(st.kbar[:, :, j_done], codebooks))
    qr = rope_at(q_t, t, p.rope_base)                                # [B, Hq, D]
    qcodes, qmargin = probe_codes(qr, codebooks, p.probes)
    qscale = code_scale(qr, codebooks)
    B, Hq, D = qr.shape
    g = Hq // p.Hkv
    j = t // p.block
    sel_own = np.empty((B, Hq, p.R + p.L), dtype=np.int64)
    smargin = np.empty((B, Hq))
    ncand = np.empty((B, Hq), dtype=np.int64)
    sscale = np.zeros((B, Hq))
    out = np.empty((B, Hq, v_t.shape[-1]))
    for b in range(B):
        for hq in range(Hq):
            h = hq // g
            row = route_row(qr[b, hq], st.kbar[b, h], probe_addresses(qcodes[b, hq], p.K),
                            st.lists[b, h], j, p.R, p.L)
            sel_own[b, hq], smargin[b, hq], ncand[b, hq] = row.sel, row.margin, row.cand.size
            sscale[b, hq] = row.scale
            use = row.sel if sel is None else np.asarray(sel[b, hq], dtype=np.int64)
            toks = selected_tokens(use, p.block)
            toks = toks[toks <= t]
            s = (st.kr[b, toks, h] @ qr[b, hq]) * p.softmax_scale
            w = np.exp(s - s.max())
            out[b, hq] = (w @ st.v[b, toks, h]) / w.sum()
    st.t = t + 1
    return DecodeOut(out, sel_own, smargin, qcodes, qmargin, ncand, qscale, sscale, *key)


# ------------------------------------------------------ 8. codebook calibration
# Spherical codebook calibration ("Monodratic: a reproducible sparse attention
# mixer", section Capacity and Figure 3: codebooks calibrated on a training
# split remove the held-out overflow and lower the maximum assigned load).
# The pages name the method and not its steps; the plainest reading is
# spherical k-means run per subspace on the routing records (post-RoPE block
# summaries, flattened), starting from the given codebooks:
#   * assign: record x goes to the codeword k maximising <x_s, C[s,k]> --
#     exactly the code assignment of section 3 (float32 scores, lower index
#     on equal scores; the argmax does not depend on |x_s|);
#   * update: C[s,k] becomes the normalised sum of the unit vectors
#     x_s/|x_s| of its members (records with x_s = 0 have no direction and
#     are left out); a codeword with no member, or whose members sum to zero,
#     keeps its value.
@dataclass
class CalibStep:
    codebooks: np.ndarray    # [P,K,dsub] float64, unit rows
    assign: np.ndarray       # [N,P] codeword of each record per subspace
    margin: np.ndarray       # [N,P] float32 gap between the best and second-best score
    counts: np.ndarray       # [P,K] members with a direction (x_s != 0)


def calibration_step(records: np.ndarray, codebooks: np.ndarray) -> CalibStep:
    """One round of spherical k-means in every subspace.  records: [N,D]
    (the values the calibration reads, float32 on the GPU); codebooks:
    [P,K,D/P]."""
    X = np.asarray(records, dtype=np.float64)
    C = np.asarray(codebooks, dtype=np.float64)
    P, K, dsub = C.shape
    N = X.shape[0]
    _, assign, margin = assign_codes(X.reshape(1, 1, N, P * dsub), C)
    assign, margin = assign[0, 0], margin[0, 0]
    new = C.copy()
    counts = np.zeros((P, K), dtype=np.int64)
    for s in range(P):
        Xs = X[:, s * dsub:(s + 1) * dsub]
        norm = np.linalg.norm(Xs, axis=1)
        for k in range(K):
            members = (assign[:, s] == k) & (norm > 0)
            counts[s, k] = members.sum()
            if counts[s, k] == 0:
                continue
            total = (Xs[members] / norm[members, None]).sum(axis=0)
            tn = np.linalg.norm(total)
            if tn > 0:
                new[s, k] = total / tn
    return CalibStep(new, assign, margin, counts)


def calibrate(records: np.ndarray, codebooks: np.ndarray, iters: int) -> np.ndarray:
    """iters rounds of calibration_step, each starting from the previous
    round's codebooks rounded to float32 (the storage type of codebooks)."""
    C = np.asarray(codebooks, dtype=np.float32)
    for _ in range(iters):
        C = calibration_step(records, C).codebooks.astype(np.float32)
    return C


def spherical_objective(records: np.ndarray, codebooks: np.ndarray) -> float:
    """Sum over records and subspaces of the cosine between x_s and its best
    codeword (records with x_s = 0 contribute nothing) -- the quantity
    spherical k-means does not decrease."""
    X = np.asarray(records, dtype=np.float64)
    C = np.asarray(codebooks, dtype=np.float64)
    P, K, dsub = C.shape
    tot = 0.0
    for s in range(P):
        Xs = X[:, s * dsub:(s + 1) * dsub]
        n = np.linalg.norm(Xs, axis=1)
        ok = n > 0
        tot += float((Xs[ok] / n[ok, None] @ C[s].T).max(axis=1).sum())
    return tot


# ---------------------------------------------------------------- 9. backward
# Gradients of the mixer's output with the route held fixed.  The Article
# ("The 99.35 Percent Result Does Not Establish Language Quality") notes that
# hard top-k choices give no ordinary gradient through the chosen index and
# leaves surrogates to the trainer; so the plainest backward differentiates
# the selected-set softmax and the rotary embedding only: given dL/d(out),
# it returns dL/dq, dL/dk, dL/dv, and nothing reaches the codebooks or the
# block summaries.
def attend_backward(qr, kr, v, sel, bs: int, scale: float, dout, rows=None, saved_out=None):
    """dL/dq', dL/dk', dL/dv of attend() for dL/d(out) = dout [B,S,Hq,D].

    Per query block j and head hq, with T = the tokens of the selected
    blocks, S = scale * q' k'^T masked to s <= t and P = softmax(S):
      dv[T]  += P^T dout_j
      dP      = dout_j v[T]^T
      dS      = P * (dP - rowsum(P * dP))
      dq'_j   = scale * dS k'[T]
      dk'[T] += scale * dS^T q'_j
    Key and value gradients of a KV head add over its query heads.  A query
    block with no valid selected block has a zero output and gets zero
    gradients.  rows: optional list of (b, hq, j) to include (dq of the
    others stays 0, and dk, dv hold only the listed rows' contributions --
    exact for a key block whose selecting rows are all listed).
    saved_out: optional [B,S,Hq,D] output saved by a forward; the row term
    rowsum(P * dP) = <dout_t, out_t> is then taken from it (equal to the
    above when the saved output is attend()'s own; a rounded copy gives the
    gradient a backward reusing that copy computes)."""
    B, S, Hq, D = qr.shape
    Hkv = kr.shape[2]
    g = Hq // Hkv
    dq = np.zeros_like(qr, dtype=np.float64)
    dk = np.zeros(kr.shape, dtype=np.float64)
    dv = np.zeros(v.shape, dtype=np.float64)
    nb = S // bs
    todo = rows if rows is not None else itertools.product(range(B), range(Hq), range(nb))
    for b, hq, j in todo:
        h = hq // g
        toks = selected_tokens(sel[b, hq, j], bs)
        if toks.size == 0:
            continue
        qpos = np.arange(j * bs, (j + 1) * bs)
        Q, Kt, Vt = qr[b, qpos, hq], kr[b, toks, h], v[b, toks, h]
        s = (Q @ Kt.T) * scale
        s[toks[None, :] > qpos[:, None]] = -np.inf
        s -= s.max(axis=1, keepdims=True)
        P = np.exp(s)
        P /= P.sum(axis=1, keepdims=True)
        dO = dout[b, qpos, hq]
        dv[b, toks, h] += P.T @ dO
        dP = dO @ Vt.T
        if saved_out is None:
            delta = (P * dP).sum(axis=1, keepdims=True)
        else:
            delta = (dO * saved_out[b, qpos, hq]).sum(axis=1, keepdims=True)
        dS = P * (dP - delta)
        dq[b, qpos, hq] = scale * dS @ Kt
        dk[b, toks, h] += scale * dS.T @ Q
    return dq, dk, dv


def rope_transpose(y: np.ndarray, base: float) -> np.ndarray:
    """The transpose of the rotation of section 1 at every position (it is
    orthogonal, so this is its inverse): y1*cos + y2*sin, y2*cos - y1*sin."""
    B, S, H, D = y.shape
    th = rope_angles(S, D, base).astype(np.float64)
    c, s = np.cos(th)[None, :, None, :], np.sin(th)[None, :, None, :]
    y1, y2 = y[..., : D // 2], y[..., D // 2:]
    return np.concatenate([y1 * c + y2 * s, y2 * c - y1 * s], axis=-1)


def backward(q, k, v, codebooks, p: Params, dout, sel=None):
    """dL/dq, dL/dk, dL/dv of forward() for dL/d(out) = dout, with the route
    of forward() (or the given sel) held fixed.  -> (dq, dk, dv, sel)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if sel is None:
        sel = forward(q, k, v, codebooks, p, attention=False).sel
    qr, kr = rope(q, p.rope_base), rope(k, p.rope_base)
    dqr, dkr, dv = attend_backward(qr, kr, v, sel, p.block, p.softmax_scale, np.asarray(dout, dtype=np.float64))
    return rope_transpose(dqr, p.rope_base), rope_transpose(dkr, p.rope_base), dv, sel
