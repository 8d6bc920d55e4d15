"""GPU parity of mdr_attend_backward (gradients of the attention output
with the route held fixed) against the oracle's attend_backward and
rope_transpose on the same seeded inputs.  The route is the oracle's; both
sides take the same sel.

Bar: the GPU works in float32 on the stored values (bfloat16 inputs are
exact in float32, and q', k' are rotated in float32 rather than rounded to
the storage type), so both dtypes are held to the same bound: for each of
dq, dk, dv, max |gpu - oracle| <= 1e-4 * max |oracle|.  Each gradient is a
float32 sum of at most a few thousand terms whose weights come from expf of
scores of size <= ~50 (relative error ~50 * 2^-24 each), so the expected
error is ~1e-5 of the largest gradient; a wrong term or index is O(1)."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from workloads import AR, CAPACITY, SCALING_32K, TINY, make_grad, make_inputs

pytestmark = pytest.mark.gpu
TOL_REL = 1e-4


def _dev(x, w):
    import torch
    if w.dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def gpu_backward(w, inp, dout_store, sel):
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    q, k, v = (_dev(x, w) for x in (inp.q_store, inp.k_store, inp.v_store))
    do = _dev(dout_store, w)
    s = torch.from_numpy(np.ascontiguousarray(sel, dtype=np.int32)).cuda()
    dq = torch.full(q.shape, np.nan, dtype=torch.float32, device="cuda")
    dk = torch.full(k.shape, np.nan, dtype=torch.float32, device="cuda")
    dv = torch.full(v.shape, np.nan, dtype=torch.float32, device="cuda")
    ws = mdr.backward_workspace(cfg)
    mdr.mdr_attend_backward(cfg, q, k, v, s, do, dq, dk, dv, ws)
    status = mdr.mdr_read_device_status(ws)
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), status


def oracle_backward(w, inp, dout, sel, rows=None):
    p = O.Params.of(w)
    qr, kr = O.rope(inp.q.astype(np.float64), p.rope_base), O.rope(inp.k.astype(np.float64), p.rope_base)
    dqr, dkr, dv = O.attend_backward(qr, kr, inp.v.astype(np.float64), sel, w.block, p.softmax_scale,
                                     dout.astype(np.float64), rows)
    return O.rope_transpose(dqr, p.rope_base), O.rope_transpose(dkr, p.rope_base), dv


def _close(name, got, ref, mask=None):
    if mask is not None:
        got, ref = got[mask], ref[mask]
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max()
    assert np.isfinite(got).all(), name
    assert err <= TOL_REL * scale, f"{name}: max error {err:.3g} > {TOL_REL} * {scale:.3g}"


@pytest.mark.parametrize("w", [TINY, AR.with_(B=4), CAPACITY, TINY.with_(R=0, L=2)],
                         ids=["tiny", "ar", "capacity_gqa", "tiny_local_only"])
def test_backward_matches_oracle(w):
    inp = make_inputs(w, 7)
    dout, dout_store = make_grad(w, 8)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel
    dq, dk, dv, status = gpu_backward(w, inp, dout_store, sel)
    assert status == 0
    rq, rk, rv = oracle_backward(w, inp, dout, sel)
    _close("dq", dq, rq)
    _close("dk", dk, rk)
    _close("dv", dv, rv)


def test_backward_caller_selection_edge_cases():
    """A row with no valid block gets zero dq and adds nothing; an id later
    than its query block is skipped and sets status 2 (the oracle's causal
    mask gives it zero weight); two runs are bit-identical."""
    w = TINY
    inp = make_inputs(w, 9)
    dout, dout_store = make_grad(w, 10)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel.copy()
    sel[0, 0, 3] = -1
    sel[0, 0, 2, 0] = 4                                   # later than block 2
    a = gpu_backward(w, inp, dout_store, sel)
    b = gpu_backward(w, inp, dout_store, sel)
    assert a[3] == 2
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_array_equal(x, y)
    assert (a[0][0, 3 * w.block:4 * w.block, 0] == 0).all()
    rq, rk, rv = oracle_backward(w, inp, dout, sel)
    _close("dq", a[0], rq)
    _close("dk", a[1], rk)
    _close("dv", a[2], rv)


def test_backward_full_size_sampled():
    """The 32K workload: dq of sampled query blocks, dk and dv of sampled
    key blocks (the oracle adds the contributions of every row that selected
    them)."""
    w = SCALING_32K
    inp = make_inputs(w, 11)
    dout, dout_store = make_grad(w, 12)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel
    dq, dk, dv, status = gpu_backward(w, inp, dout_store, sel)
    assert status == 0
    r = np.random.default_rng(13)
    qrows = [(0, int(r.integers(w.Hq)), int(j)) for j in (0, 1, w.nb - 1, *r.integers(2, w.nb - 1, size=5))]
    keys = [(0, int(r.integers(w.Hkv)), int(i)) for i in (0, w.nb - 1, *r.integers(1, w.nb - 1, size=3))]
    g = w.Hq // w.Hkv
    rows = set(qrows)
    for b, h, i in keys:
        for hq in range(h * g, (h + 1) * g):
            for j in range(w.nb):
                if i in sel[b, hq, j]:
                    rows.add((b, hq, j))
    rq, rk, rv = oracle_backward(w, inp, dout, sel, sorted(rows))
    qmask = np.zeros(dq.shape[:3], dtype=bool)
    for b, hq, j in qrows:
        qmask[b, j * w.block:(j + 1) * w.block, hq] = True
    kmask = np.zeros(dk.shape[:3], dtype=bool)
    for b, h, i in keys:
        kmask[b, i * w.block:(i + 1) * w.block, h] = True
    _close("dq", dq, rq, qmask)
    _close("dk", dk, rk, kmask)
    _close("dv", dv, rv, kmask)
