"""GPU parity of mdr_attend_backward (gradients of the attention output
with the route held fixed) against the oracle's attend_backward and
rope_transpose on the same seeded inputs.  The route is the oracle's; both
sides take the same sel.

Bar, float32 storage (CUDA cores, float32 on the stored values): for each
of dq, dk, dv, max |gpu - oracle| <= 1e-4 * max |oracle|.  Each gradient is a
float32 sum of at most a few thousand terms whose weights come from expf of
scores of size <= ~50 (relative error ~50 * 2^-24 each), so the expected
error is ~1e-5 of the largest gradient; a wrong term or index is O(1).

Bar, bfloat16 storage (tensor cores): the products take bfloat16 operands --
the rotated q', k' (as in the forward) and the weights P and dS -- each
rounded with relative error <= 2^-9, accumulated in float32.  A gradient row
is a sum of such products, so its error relative to its terms is a few
times 2^-9 ~ 1e-2, the bfloat16 tolerance of the forward (2e-2 relative).
For each of dq, dk, dv and every row (token, head):
  ||gpu - oracle||_2 <= 2e-2 * max(||oracle row||_2, rms row norm),
the floor at the tensor's root-mean-square row norm covering rows whose
dS = P (dP - Delta) cancels (a small difference of O(1) terms; a token that
sees a single key has dS = 0 exactly in the oracle and ~1e-8 on the GPU);
rows that are zero by construction (a query block with no selected block, a
key block no query block selected) are exactly zero on the GPU; and
max |gpu - oracle| <= 2e-2 * max |oracle|."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from workloads import AR, CAPACITY, SCALING_32K, TINY, make_grad, make_inputs, scaling

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
    if status != 0:      # the second word says where a tensor-core CTA gave up
        print(f"backward status {status}, site {int(ws[:16].view(torch.int32)[1].item())}")
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy(), status


def oracle_backward(w, inp, dout, sel, rows=None, saved_out=None):
    p = O.Params.of(w)
    qr, kr = O.rope(inp.q.astype(np.float64), p.rope_base), O.rope(inp.k.astype(np.float64), p.rope_base)
    dqr, dkr, dv = O.attend_backward(qr, kr, inp.v.astype(np.float64), sel, w.block, p.softmax_scale,
                                     dout.astype(np.float64), rows, saved_out)
    return O.rope_transpose(dqr, p.rope_base), O.rope_transpose(dkr, p.rope_base), dv


TOL_BF16 = 2e-2


def structural_zeros(w, sel):
    """Rows whose gradient is zero by construction, not by cancellation: dq
    of query blocks with no valid selected block; dk, dv of key blocks no
    query block selected.  -> (dq mask [B,S,Hq], dk/dv mask [B,S,Hkv])."""
    B, Hq, nb, _ = sel.shape
    g = Hq // w.Hkv
    j = np.arange(nb)[None, None, :, None]
    valid = (sel >= 0) & (sel <= j)
    qz = ~valid.any(axis=-1)                                   # [B,Hq,nb]
    used = np.zeros((B, w.Hkv, nb), dtype=bool)
    for b, hq, jj, n in zip(*np.nonzero(valid)):
        used[b, hq // g, sel[b, hq, jj, n]] = True
    rep = lambda m: np.repeat(m.transpose(0, 2, 1), w.block, axis=1)
    return rep(qz), rep(~used)


def _close(name, got, ref, mask=None, dtype="f32", zeros=None):
    """got, ref [B,S,H,D]; mask [B,S,H] selects the rows compared; zeros
    [B,S,H] marks rows that must be exactly zero (structural_zeros)."""
    if zeros is not None:
        assert (got[zeros] == 0).all(), f"{name}: rows that are zero by construction are not zero"
    if mask is not None:
        got, ref = got[mask], ref[mask]
    else:
        got, ref = got.reshape(-1, got.shape[-1]), ref.reshape(-1, ref.shape[-1])
    assert np.isfinite(got).all(), name
    scale = max(np.abs(ref).max(), 1e-30)
    err = np.abs(got - ref).max()
    if dtype == "f32":
        assert err <= TOL_REL * scale, f"{name}: max error {err:.3g} > {TOL_REL} * {scale:.3g}"
        return err / scale
    assert err <= TOL_BF16 * scale, f"{name}: max error {err:.3g} > {TOL_BF16} * {scale:.3g}"
    rn = np.linalg.norm(ref, axis=-1)
    rms = np.sqrt(np.mean(rn ** 2))
    rel = np.linalg.norm(got - ref, axis=-1) / np.maximum(rn, rms)
    assert rel.max() <= TOL_BF16, f"{name}: row error {rel.max():.3g} > {TOL_BF16} (row {int(rel.argmax())})"
    return float(rel.max())


CASES = {
    "tiny": TINY,                                               # float32, CUDA cores
    "tiny_local_only": TINY.with_(R=0, L=2),
    "ar": AR.with_(B=4),                                        # bf16, block 64, D 64
    "capacity_gqa": CAPACITY,                                   # bf16, block 64, D 64, 3 query heads per KV head
    "scaling4k": scaling(4096),                                 # bf16, block 64, D 128
    "ragged_gqa_b128_d64": CAPACITY.with_(S=7 * 128, block=128, Hq=6, Hkv=2, R=3, L=3, keys="gaussian"),
    "b128_d128": CAPACITY.with_(S=1024, block=128, D=128, Hq=4, Hkv=2, R=3, L=2, K=8, keys="gaussian"),
    "local_only_bf16": AR.with_(B=2, R=0, L=2),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name):
    w = CASES[name]
    inp = make_inputs(w, 7)
    dout, dout_store = make_grad(w, 8)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel
    dq, dk, dv, status = gpu_backward(w, inp, dout_store, sel)
    assert status == 0
    rq, rk, rv = oracle_backward(w, inp, dout, sel)
    qz, kz = structural_zeros(w, sel)
    errs = [_close(n, x, y, dtype=w.dtype, zeros=z)
            for n, x, y, z in (("dq", dq, rq, qz), ("dk", dk, rk, kz), ("dv", dv, rv, kz))]
    print(f"backward {name}: {errs}")


def test_backward_caller_selection_edge_cases_bf16():
    """Tensor-core path: a row with no valid block gets zero dq and adds
    nothing; an id later than its query block is skipped and sets status 2;
    two runs are bit-identical."""
    w = AR.with_(B=2)
    inp = make_inputs(w, 19)
    dout, dout_store = make_grad(w, 20)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel.copy()
    sel[0, 1, 3] = -1
    sel[1, 2, 2, 0] = 4                                   # later than block 2
    a = gpu_backward(w, inp, dout_store, sel)
    b = gpu_backward(w, inp, dout_store, sel)
    assert a[3] == 2
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_array_equal(x, y)
    assert (a[0][0, 3 * w.block:4 * w.block, 1] == 0).all()
    rq, rk, rv = oracle_backward(w, inp, dout, sel)
    qz, kz = structural_zeros(w, sel)
    assert qz[0, 3 * w.block:4 * w.block, 1].all()
    _close("dq", a[0], rq, dtype="bf16", zeros=qz)
    _close("dk", a[1], rk, dtype="bf16", zeros=kz)
    _close("dv", a[2], rv, dtype="bf16", zeros=kz)


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
    errs = [_close("dq", dq, rq, qmask, w.dtype), _close("dk", dk, rk, kmask, w.dtype),
            _close("dv", dv, rv, kmask, w.dtype)]
    print(f"backward {w.name} sampled: {errs}")


def gpu_attend_train(w, inp, sel):
    """mdr_attend_train on the given selection: the output (device tensor in
    the storage type) and the row normalisers (numpy [B,Hq,S])."""
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    q, k, v = (_dev(x, w) for x in (inp.q_store, inp.k_store, inp.v_store))
    s = torch.from_numpy(np.ascontiguousarray(sel, dtype=np.int32)).cuda()
    out = torch.empty_like(q)
    lse = torch.full((w.B, w.Hq, w.S), np.nan, dtype=torch.float32, device="cuda")
    ws = mdr.workspace(cfg)
    mdr.mdr_attend_train(cfg, q, k, v, s, out, lse, ws)
    assert mdr.mdr_read_device_status(ws) == 0
    return out, lse.cpu().numpy()


@pytest.mark.parametrize("name", sorted(CASES))
def test_forward_lse_matches_oracle(name):
    """The row normalisers written with the forward output (per-head tiles,
    grouped-query units at block 128, float32 rows) against the oracle's.
    Bar: |gpu - oracle| <= 2^-7 * scale * |q'_t| * max_s |k'_s| per
    row: the normaliser moves by at most the largest change of a score, and
    a bf16 q' or k' moves a score by at most 2^-8 of that product; plus
    2e-5 + 2e-6 |lse| for the float32 sums and logarithm."""
    w = CASES[name]
    inp = make_inputs(w, 31)
    p = O.Params.of(w)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, p, attention=False).sel
    _, lse = gpu_attend_train(w, inp, sel)
    qr, kr = O.rope(inp.q.astype(np.float64), p.rope_base), O.rope(inp.k.astype(np.float64), p.rope_base)
    ref = O.softmax_lse(qr, kr, sel, w.block, p.softmax_scale)
    assert np.isneginf(ref).sum() == np.isneginf(lse).sum() and (np.isneginf(ref) == np.isneginf(lse)).all()
    fin = np.isfinite(ref)
    qn = np.linalg.norm(qr, axis=-1).transpose(0, 2, 1)                      # [B,Hq,S]
    kmax = np.linalg.norm(kr, axis=-1).max()
    tol = (2.0 ** -7 * p.softmax_scale * qn * kmax if w.dtype == "bf16" else 0.0) + 2e-5 + 2e-6 * np.abs(
        np.where(fin, ref, 0.0))
    err = np.abs(lse - ref)
    assert (err[fin] <= tol[fin]).all(), f"{name}: worst lse error {err[fin].max():.3g}"
    print(f"lse {name}: max error {err[fin].max():.3g}")


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_saved_matches_oracle(name):
    """mdr_attend_backward_saved, fed the output and row normalisers of
    mdr_attend_train on the same selection (tensor cores: no statistics
    pass), against the oracle's gradients given that saved output, at the
    same bar as the backward that recomputes them.  (Against the exact
    output the row term <dout_t, out_t> carries the output's bf16 rounding,
    2^-9 of sum_d |dout_td out_td|, which dS = P (dP - Delta) can magnify
    where dP and Delta nearly cancel.)"""
    import torch
    from learned_product_hash_b200 import mdr
    w = CASES[name]
    inp = make_inputs(w, 7)
    dout, dout_store = make_grad(w, 8)
    sel = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False).sel
    out, lse = gpu_attend_train(w, inp, sel)
    cfg = mdr.make_config(w)
    q, k, v = (_dev(x, w) for x in (inp.q_store, inp.k_store, inp.v_store))
    do = _dev(dout_store, w)
    s = torch.from_numpy(np.ascontiguousarray(sel, dtype=np.int32)).cuda()
    dq = torch.full(q.shape, np.nan, dtype=torch.float32, device="cuda")
    dk = torch.full(k.shape, np.nan, dtype=torch.float32, device="cuda")
    dv = torch.full(v.shape, np.nan, dtype=torch.float32, device="cuda")
    ws = mdr.backward_workspace(cfg)
    mdr.mdr_attend_backward_saved(cfg, q, k, v, s, out, torch.from_numpy(lse).cuda(), do, dq, dk, dv, ws)
    assert mdr.mdr_read_device_status(ws) == 0
    # The reference is the gradient given the saved output: the oracle takes
    # <dout_t, out_t> from the GPU forward's (rounded) output, as the kernel does.
    saved = out.float().cpu().numpy().astype(np.float64)
    rq, rk, rv = oracle_backward(w, inp, dout, sel, saved_out=saved)
    qz, kz = structural_zeros(w, sel)
    errs = [_close(n, x.cpu().numpy(), y, dtype=w.dtype, zeros=z)
            for n, x, y, z in (("dq", dq, rq, qz), ("dk", dk, rk, kz), ("dv", dv, rv, kz))]
    print(f"backward saved {name}: {errs}")
