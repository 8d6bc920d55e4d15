"""The GPU parity harness (tests/parity_util.compare) on the CPU: outputs
that take a near-tie decision the other way must pass, with what follows from
that choice checked against the oracle re-run with it; outputs that differ
outside a near tie must fail.  The "GPU" side here is the oracle itself, run
with a decision forced, so no GPU is needed."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import parity_util as U
from workloads import TINY, make_inputs


def _as_gpu(res, w):
    """The fields run_gpu returns, from an oracle result."""
    return {"status": 0, "kbar": res.kbar.astype(np.float32), "qbar": res.qbar.astype(np.float32),
            "addr": res.addr.copy(), "lists": res.lists.copy(), "load": res.load.copy(),
            "overflow": res.overflow.copy(), "maxload": res.maxload.copy(), "sel": res.sel.copy(),
            "qcodes": res.qcodes.copy(), "ncand": res.ncand.copy(), "out": res.out.astype(np.float32)}


def _tied_case(seed=0):
    """TINY with one subspace-0 codeword copied over another: every block
    whose best subspace-0 codeword is the copied one holds an exact tie
    between the two, and the oracle takes the lower index LO (HI is the other
    valid choice).  The copied codeword is the most common key code."""
    w = TINY.with_(S=192, R=3, L=1, cap=3)
    inp = make_inputs(w, seed)
    p = O.Params.of(w)
    res0 = O.forward(inp.q, inp.k, inp.v, inp.codebooks, p, attention=False)
    c = int(np.bincount(res0.codes[..., 0].ravel(), minlength=w.K).argmax())
    d = (c + 3) % w.K
    cb = inp.codebooks.copy()
    cb[0, d] = cb[0, c]
    res = O.forward(inp.q, inp.k, inp.v, cb, p)
    return w, inp, cb, p, res, min(c, d), max(c, d)


def test_exact_equality_passes():
    w, inp, cb, p, res, LO, HI = _tied_case()
    rep = U.compare(w, _as_gpu(res, w), res, cb, max_ties=0)
    assert rep["code_ties"] == rep["qcode_ties"] == rep["sel_ties"] == rep["rerun_rows"] == 0


def test_tied_key_code_taken_the_other_way_passes():
    w, inp, cb, p, res, LO, HI = _tied_case()
    tied = res.codes[..., 0] == LO
    assert tied.sum() >= 2, "the case must hold ties"
    addr = res.addr.copy()
    addr[tied] += (HI - LO) * w.K                                 # subspace 0 is the most significant
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, addr=addr)
    g = _as_gpu(alt, w)
    assert not np.array_equal(g["lists"], res.lists)
    rep = U.compare(w, g, res, cb)
    assert rep["code_ties"] == int(tied.sum())
    assert rep["rerun_rows"] == int((alt.sel != res.sel).any(axis=-1).sum())


def test_tied_probe_taken_the_other_way_passes():
    w, inp, cb, p, res, LO, HI = _tied_case(1)
    qc = res.qcodes.copy()
    hit = (qc[..., 0, :] == LO).any(axis=-1) & ~(qc[..., 0, :] == HI).any(axis=-1)
    assert hit.any(), "the case must hold probe ties"
    sub0 = qc[..., 0, :]
    sub0[hit[..., None] & (sub0 == LO)] = HI
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, qcodes=qc)
    rep = U.compare(w, _as_gpu(alt, w), res, cb)
    assert rep["qcode_ties"] == int(hit.sum())


def test_code_differing_outside_a_tie_fails():
    w, inp, cb, p, res, LO, HI = _tied_case()
    addr = res.addr.copy()
    b, h, n = np.argwhere(res.codes[..., 1] != (res.codes[..., 1] + 1) % w.K)[0]
    addr[b, h, n] = res.codes[b, h, n, 0] * w.K + (res.codes[b, h, n, 1] + 1) % w.K
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, addr=addr)
    with pytest.raises(AssertionError, match="key codes differ outside near ties"):
        U.compare(w, _as_gpu(alt, w), res, cb)


def test_route_differing_outside_a_tie_fails():
    w = TINY.with_(S=192, K=4, probes=4, cap=12, R=2, L=1)       # every eligible block a candidate
    inp = make_inputs(w, 2)
    cb, p = inp.codebooks, O.Params.of(w)
    res = O.forward(inp.q, inp.k, inp.v, cb, p)
    sel = res.sel.copy()
    idx = np.argwhere((res.ncand > w.R) & ~O.near_tie(res.sel_margin, res.sel_scale))[0]
    b, hq, j = idx
    row = O.route_row(res.qbar[b, hq, j], res.kbar[b, 0], O.probe_addresses(res.qcodes[b, hq, j], w.K),
                      res.lists[b, 0], j, w.R, w.L)
    loser = [i for i in row.cand.tolist() if i not in sel[b, hq, j]][0]
    remote = sorted(sel[b, hq, j, : w.R].tolist()[1:] + [loser])
    sel[b, hq, j, : w.R] = remote
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, sel=sel)
    with pytest.raises(AssertionError, match="routes differ outside near ties"):
        U.compare(w, _as_gpu(alt, w), res, cb)


def test_attention_of_a_rerun_row_is_checked():
    """A tied code taken the other way changes routes; the attention of those
    rows is compared with the oracle on the new selection, so an output that
    kept the old selection's attention fails."""
    w, inp, cb, p, res, LO, HI = _tied_case()
    tied = res.codes[..., 0] == LO
    addr = res.addr.copy()
    addr[tied] += (HI - LO) * w.K
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, addr=addr)
    changed = (alt.sel != res.sel).any(axis=-1)
    assert changed.any()
    g = _as_gpu(alt, w)
    g["out"] = res.out.astype(np.float32)                         # attention of the old selection
    with pytest.raises(AssertionError, match="max abs error"):
        U.compare(w, g, res, cb)


def test_tie_budget():
    w, inp, cb, p, res, LO, HI = _tied_case()
    tied = res.codes[..., 0] == LO
    addr = res.addr.copy()
    addr[tied] += (HI - LO) * w.K
    alt = O.forward(inp.q, inp.k, inp.v, cb, p, addr=addr)
    with pytest.raises(AssertionError, match="budget"):
        U.compare(w, _as_gpu(alt, w), res, cb, max_ties=1)
