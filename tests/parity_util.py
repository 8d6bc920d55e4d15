"""Helpers for the GPU parity tests: run the CUDA library through its C ABI
on seeded inputs and compare with the CPU oracle.

The bar (stated once here, used by every parity test):
  * codes, posting lists, loads, overflow, max load, probed codewords,
    candidate counts and selected block ids: bit-exact.  A routing decision
    whose float32 margin in the oracle is below 1e-6*max(1,|s|) is a near tie:
    there either choice is correct, the GPU's choice must be one of the tied
    ones, and outputs downstream of it are checked for validity instead.
  * summaries (float32): |gpu - oracle| <= 1e-5 + 1e-5*|oracle|.
  * attention output: float32 storage, max |gpu - oracle| <= 1e-5; bfloat16
    storage, for every output row (token, head) ||gpu - oracle||_2 <=
    2e-2 * ||oracle||_2, and max |gpu - oracle| <= 2e-2 * max |oracle|.
    (bfloat16 operands alone -- the rotated q', k' rounded to bfloat16 --
    put about 1e-2 into the worst row of the planted-block workload, whose
    scores are large.)
"""
from __future__ import annotations

import numpy as np

from oracle import mdr_oracle as O
from workloads import make_inputs

TOL_F32_OUT = 1e-5
TOL_BF16_REL = 2e-2


def to_device(inp, w):
    import torch
    def t(x):
        if w.dtype == "bf16":
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        return torch.from_numpy(x).cuda()
    return t(inp.q_store), t(inp.k_store), t(inp.v_store), torch.from_numpy(inp.codebooks).cuda()


def out_to_numpy(out, w):
    import torch
    return out.float().cpu().numpy()


def run_gpu(w, inp, entry="forward", force=None):
    """entry "forward" = mdr_forward; "split" = mdr_build_index + mdr_route +
    mdr_attend; "forced" = the split path with mdr_route_forced and the
    forced ids ``force`` [B,Hq,nb]."""
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    q, k, v, cb = to_device(inp, w)
    idx = mdr.Index.empty(cfg)
    rt = mdr.RouteOut.empty(cfg, debug=True)
    out = torch.empty_like(q)
    ws = mdr.workspace(cfg)
    if entry == "forward":
        mdr.mdr_forward(cfg, q, k, v, cb, idx, rt, out, ws)
    else:
        mdr.mdr_build_index(cfg, k, cb, idx, ws)
        if entry == "forced":
            f = torch.from_numpy(np.ascontiguousarray(force, dtype=np.int32)).cuda()
            mdr.mdr_route_forced(cfg, q, cb, idx, f, rt, ws)
        else:
            mdr.mdr_route(cfg, q, cb, idx, rt, ws)
        mdr.mdr_attend(cfg, q, k, v, rt.sel, out, ws)
    status = mdr.mdr_read_device_status(ws)
    torch.cuda.synchronize()
    g = {f: getattr(idx, f).cpu().numpy() for f in ("kbar", "addr", "lists", "load", "overflow", "maxload")}
    g.update({f: getattr(rt, f).cpu().numpy() for f in ("sel", "qbar", "qcodes", "ncand")})
    g["out"] = out_to_numpy(out, w)
    g["status"] = status
    return g


def check_out(w, got, ref, mask_rows=None):
    """Compare attention outputs [B,S,Hq,D]; NaN rows of ref are skipped."""
    ok = ~np.isnan(ref[..., 0])
    if mask_rows is not None:
        ok &= mask_rows
    g, r = got[ok], ref[ok]
    if g.size == 0:
        return 0.0
    if w.dtype == "f32":
        err = np.abs(g - r).max()
        assert err <= TOL_F32_OUT, f"max abs error {err:.3g} > {TOL_F32_OUT}"
        return float(err)
    rel = np.linalg.norm(g - r, axis=-1) / np.linalg.norm(r, axis=-1)
    assert rel.max() <= TOL_BF16_REL, f"max row relative error {rel.max():.3g} > {TOL_BF16_REL}"
    glob = np.abs(g - r).max() / np.abs(r).max()
    assert glob <= TOL_BF16_REL, f"max abs error {glob:.3g} of max |out| > {TOL_BF16_REL}"
    return float(rel.max())


def valid_lists(lists, load, addr, cap, nb):
    """Invariants of one head's lists (used where a near tie changed codes)."""
    A = lists.shape[0]
    stored = lists[lists >= 0]
    assert stored.size == np.unique(stored).size
    for a in range(A):
        row = lists[a]
        n = int((row >= 0).sum())
        assert n == min(load[a], cap) and (row[:n] >= 0).all() and (row[n:] == -1).all()
        assert np.all(np.diff(row[:n]) > 0)
        assert all(addr[i] == a for i in row[:n])


def compare(w, g, res, codebooks):
    """Compare GPU outputs g with the oracle result res.  Returns a report."""
    rep = {"code_ties": 0, "qcode_ties": 0, "sel_ties": 0}
    assert g["status"] == 0, f"device status {g['status']}"
    np.testing.assert_allclose(g["kbar"], res.kbar, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(g["qbar"], res.qbar, rtol=1e-5, atol=1e-5)

    # key codes
    best = np.max(np.abs(O.codeword_scores(res.kbar, codebooks)), axis=-1)
    tie_k = O.near_tie(res.code_margin, best).any(axis=-1)            # [B,Hkv,nb]
    diff_k = g["addr"] != res.addr
    assert not (diff_k & ~tie_k).any(), f"{int((diff_k & ~tie_k).sum())} key addresses differ outside near ties"
    rep["code_ties"] = int((diff_k & tie_k).sum())
    head_same = ~diff_k.any(axis=-1)                                    # [B,Hkv]
    B, Hkv = head_same.shape
    for b in range(B):
        for h in range(Hkv):
            if head_same[b, h]:
                assert np.array_equal(g["lists"][b, h], res.lists[b, h]), (b, h)
                assert np.array_equal(g["load"][b, h], res.load[b, h]), (b, h)
                assert g["overflow"][b, h] == res.overflow[b, h] and g["maxload"][b, h] == res.maxload[b, h]
            else:
                valid_lists(g["lists"][b, h], g["load"][b, h], g["addr"][b, h], w.cap, w.nb)

    # query probes (a set per subspace)
    qbest = np.max(np.abs(O.codeword_scores(res.qbar, codebooks)), axis=-1)
    tie_q = O.near_tie(res.qcode_margin, qbest)                         # [B,Hq,nb,P]
    diff_q = (np.sort(g["qcodes"], axis=-1) != np.sort(res.qcodes, axis=-1)).any(axis=-1)
    assert not (diff_q & ~tie_q).any(), "probed codewords differ outside near ties"
    rep["qcode_ties"] = int((diff_q & tie_q).sum())

    # routes whose inputs are identical on both sides
    g_ = w.Hq // w.Hkv
    up_same = head_same[:, np.arange(w.Hq) // g_][:, :, None] & ~diff_q.any(axis=-1)
    sel_same = (g["sel"] == res.sel).all(axis=-1)
    tie_s = O.near_tie(res.sel_margin, 1.0)
    bad = up_same & ~sel_same & ~tie_s
    assert not bad.any(), f"{int(bad.sum())} routes differ outside near ties, first at {np.argwhere(bad)[0]}"
    rep["sel_ties"] = int((up_same & ~sel_same).sum())
    assert np.array_equal(g["ncand"][up_same], res.ncand[up_same])
    # every route, tied or not, obeys causality and the row layout
    R, L = w.R, w.L
    remote = g["sel"][..., :R]
    jj = np.arange(w.nb)[None, None, :, None]
    assert ((remote == -1) | ((remote >= 0) & (remote <= jj - L))).all()
    loc = np.arange(w.nb)[:, None] - L + 1 + np.arange(L)[None, :]
    assert np.array_equal(g["sel"][..., R:], np.broadcast_to(np.where(loc >= 0, loc, -1), g["sel"][..., R:].shape))

    # attention where the selection agrees
    rowmask = np.repeat(sel_same.transpose(0, 2, 1), w.block, axis=1)   # [B,S,Hq]
    rep["out_err"] = check_out(w, g["out"], res.out, rowmask)
    rep["overflow"] = int(g["overflow"].sum())
    return rep


def sampled_rows(w, res, n=12, seed=0):
    """Query blocks (b, hq, j) whose attention the oracle computes at full
    size: the first and last, the four with the most candidates, and random
    ones."""
    r = np.random.default_rng(seed)
    rows = {(0, 0, 0), (0, w.Hq - 1, w.nb - 1)}
    heavy = np.argsort(-res.ncand.ravel())[:4]
    for f in heavy:
        b, h, j = np.unravel_index(f, res.ncand.shape)
        rows.add((int(b), int(h), int(j)))
    while len(rows) < n:
        rows.add((int(r.integers(w.B)), int(r.integers(w.Hq)), int(r.integers(w.nb))))
    return sorted(rows)


def oracle_for(w, inp, rows=None, force=None):
    return O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), rows=rows, force=force)
