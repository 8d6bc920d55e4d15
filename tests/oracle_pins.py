"""Checks that pin the CPU oracle to facts other than itself.

Each check raises AssertionError when the oracle disagrees with a closed form,
an invariant the pages state, a brute-force enumeration on a tiny input, or a
library routine that computes the same textbook quantity.  The checks are
plain functions so that the mutation tests can run them against an oracle with
a planted mistake and require that at least one of them fails.

Citations: "Report" is the page "Monodratic: a reproducible sparse attention
mixer"; "Article" is the page "Monodratic Claims Learned Routing Can Make
Sparse Causal Attention More Selective".
"""
from __future__ import annotations

import itertools
import json
import os
from fractions import Fraction

import numpy as np
import torch

from oracle import mdr_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _p(**kw):
    base = dict(B=1, S=96, Hq=1, Hkv=1, D=32, block=16, P=2, K=8, cap=8,
                probes=2, R=2, L=1, rope_base=10000.0, scale=0.0)
    base.update(kw)
    return O.Params(**base)


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _unit_codebooks(P, K, d, seed):
    c = _rand((P, K, d), seed)
    return (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)


# ------------------------------------------------------------------ rotary
def check_rope_inv_freq_closed_form():
    """omega_i = base^(-2i/D): for D=4, base=100 the frequencies are 1 and 1/10."""
    w = O.rope_inv_freq(4, 100.0)
    assert w.dtype == np.float32
    assert w[0] == np.float32(1.0) and w[1] == np.float32(0.1), w


def check_rope_complex_phase():
    """Rotary embedding as multiplication of z = x_i + 1j*x_{i+D/2} by
    exp(1j*theta): the rotation written with complex numbers, independently of
    the real cos/sin form."""
    D, S = 16, 40
    x = _rand((1, S, 2, D), 1)
    xr = O.rope(x, 10000.0)
    th = O.rope_angles(S, D, 10000.0).astype(np.float64)
    z = (x[..., : D // 2] + 1j * x[..., D // 2:]) * np.exp(1j * th)[None, :, None, :]
    assert np.allclose(xr[..., : D // 2], z.real, atol=1e-12)
    assert np.allclose(xr[..., D // 2:], z.imag, atol=1e-12)
    # unit vector e_0 at position 1 with theta_0 = 1 turns to (cos 1, sin 1)
    e = np.zeros((1, 2, 1, 2))
    e[0, 1, 0, 0] = 1.0
    r = O.rope(e, 10000.0)[0, 1, 0]
    assert np.allclose(r, [np.cos(1.0), np.sin(1.0)], atol=1e-15)


def check_rope_identity_and_norms():
    D, S = 32, 50
    x = _rand((2, S, 3, D), 2)
    xr = O.rope(x, 10000.0)
    assert np.array_equal(xr[:, 0], x[:, 0]), "position 0 must be the identity"
    n0 = x[..., : D // 2] ** 2 + x[..., D // 2:] ** 2
    n1 = xr[..., : D // 2] ** 2 + xr[..., D // 2:] ** 2
    assert np.allclose(n0, n1, rtol=1e-12, atol=1e-12), "each pair keeps its length"


def check_rope_relative_position():
    """<R(t)a, R(t+d)b> depends only on d: the property that makes rotary
    scores relative.  Angles are float32 products, so it holds to their
    rounding at these small positions."""
    D, S = 32, 64
    a, b = _rand((2, D), 3)
    x = np.zeros((1, S, 1, D))
    t, d = 37, 11
    x[0, t, 0], x[0, t + d, 0], x[0, 0, 0], x[0, d, 0] = a, b, a, b
    xr = O.rope(x, 10000.0)
    lhs = xr[0, t, 0] @ xr[0, t + d, 0]
    rhs = xr[0, 0, 0] @ xr[0, d, 0]
    assert abs(lhs - rhs) < 1e-4 * max(1.0, abs(rhs)), (lhs, rhs)


# --------------------------------------------------------------- summaries
def check_block_mean_geometric_series():
    """A block whose tokens all hold the same vector c has, per rotary pair,
    the mean (1/bs) * sum_t exp(1j*theta*t) * z_c: a geometric series with a
    closed form."""
    D, bs, S = 16, 8, 48
    c = _rand((D,), 4)
    x = np.tile(c, (1, S, 1, 1))
    mean = O.block_means(O.rope(x, 10000.0), bs)          # [1,1,nb,D]
    omega = O.rope_inv_freq(D, 10000.0).astype(np.float64)
    z = c[: D // 2] + 1j * c[D // 2:]
    for j in range(S // bs):
        t0 = j * bs
        r = np.exp(1j * omega)
        with np.errstate(invalid="ignore", divide="ignore"):
            gs = np.where(np.abs(1 - r) > 0, r ** t0 * (1 - r ** bs) / (1 - r), bs)
        closed = z * gs / bs
        got = mean[0, 0, j, : D // 2] + 1j * mean[0, 0, j, D // 2:]
        assert np.allclose(got, closed, atol=2e-6), (j, np.abs(got - closed).max())


def check_block_mean_constant_blocks():
    """Blockwise-constant inputs are their own block means, and the mean is
    linear (the mean alone, on unrotated arrays)."""
    B, nb, bs, H, D = 2, 5, 4, 3, 6
    c = _rand((B, nb, H, D), 5)
    x = np.repeat(c, bs, axis=1)                    # [B, S, H, D]
    m = O.block_means(x, bs)
    assert np.allclose(m, c.transpose(0, 2, 1, 3), atol=1e-15)
    # linearity
    y = _rand(x.shape, 6)
    assert np.allclose(O.block_means(2 * x + y, bs), 2 * m + O.block_means(y, bs), atol=1e-12)


# ------------------------------------------------------------------ codes
def check_codes_single_codeword():
    """K = 1: every block gets code 0 and address 0."""
    kbar = _rand((1, 2, 7, 8), 7)
    cb = _unit_codebooks(2, 1, 4, 8)
    addr, codes, _ = O.assign_codes(kbar, cb)
    assert (addr == 0).all() and (codes == 0).all()


def check_codes_signed_basis():
    """Codebook {+e_0, -e_0, +e_1, -e_1, ...}: the best codeword is the
    coordinate of largest magnitude with its sign."""
    d, P = 4, 2
    K = 2 * d
    cb = np.zeros((P, K, d), dtype=np.float32)
    for s in range(P):
        for i in range(d):
            cb[s, 2 * i, i] = 1.0
            cb[s, 2 * i + 1, i] = -1.0
    kbar = _rand((1, 1, 50, P * d), 9)
    addr, codes, _ = O.assign_codes(kbar, cb)
    for n in range(50):
        expect = []
        for s in range(P):
            sub = kbar[0, 0, n, s * d:(s + 1) * d]
            i = int(np.argmax(np.abs(sub)))
            expect.append(2 * i + (1 if sub[i] < 0 else 0))
        assert list(codes[0, 0, n]) == expect
        assert addr[0, 0, n] == expect[0] * K + expect[1], "first subspace is most significant"


def check_codes_key_equals_codeword():
    cb = _unit_codebooks(2, 6, 5, 10)
    for a in range(6):
        for b in range(6):
            kbar = np.concatenate([cb[0, a], cb[1, b]]).astype(np.float64)[None, None, None, :]
            addr, codes, _ = O.assign_codes(kbar, cb)
            assert list(codes[0, 0, 0]) == [a, b] and addr[0, 0, 0] == a * 6 + b
    # scaling by a positive factor changes nothing; zero goes to code 0
    kbar = _rand((1, 1, 20, 10), 11)
    assert np.array_equal(O.assign_codes(kbar, cb)[0], O.assign_codes(3.7 * kbar, cb)[0])
    assert (O.assign_codes(np.zeros((1, 1, 3, 10)), cb)[0] == 0).all()


def check_probe_top_p_bruteforce():
    """The p probes per subspace are the p best codewords, found here by
    sorting (-score, index) tuples with Python's sorted()."""
    cb = _unit_codebooks(2, 8, 6, 12)
    qbar = _rand((1, 1, 30, 12), 13)
    codes, _ = O.probe_codes(qbar, cb, 3)
    for n in range(30):
        for s in range(2):
            sc = [float(np.float32(qbar[0, 0, n, 6 * s:6 * s + 6].astype(np.float32) @ cb[s, k])) for k in range(8)]
            best = [k for _, k in sorted((-v, k) for k, v in enumerate(sc))[:3]]
            assert list(codes[0, 0, n, s]) == best
    pa = O.probe_addresses(np.array([[1, 4], [2, 0]]), 8)
    assert list(pa) == [1 * 8 + 2, 1 * 8 + 0, 4 * 8 + 2, 4 * 8 + 0]


# ------------------------------------------------------------------ lists
def check_lists_single_address():
    """A = 1: the list holds blocks 0..cap-1, the rest overflow."""
    for nb, cap in [(10, 4), (3, 8), (8, 8)]:
        lists, load, ovf, mx = O.build_lists(np.zeros(nb, dtype=np.int64), 1, cap)
        exp = np.full(cap, -1)
        exp[: min(nb, cap)] = np.arange(min(nb, cap))
        assert np.array_equal(lists[0], exp)
        assert ovf == max(0, nb - cap) and mx == nb and load[0] == nb


def check_lists_stable_sort():
    """The lists equal a stable sort of the blocks by address (the report's
    index build uses a stable sort), truncated to capacity."""
    r = np.random.default_rng(14)
    for A, cap, nb in [(16, 3, 100), (64, 8, 300), (5, 50, 40)]:
        addr = r.integers(0, A, nb)
        lists, load, ovf, mx = O.build_lists(addr, A, cap)
        order = np.argsort(addr, kind="stable")
        for a in range(A):
            ids = order[addr[order] == a][:cap]
            row = np.full(cap, -1)
            row[: ids.size] = ids
            assert np.array_equal(lists[a], row)
        assert np.array_equal(load, np.bincount(addr, minlength=A))
        stored = (lists >= 0).sum()
        assert stored + ovf == nb and (lists >= 0).sum(axis=1).max() <= cap
        assert mx == load.max()
        seen = lists[lists >= 0]
        assert seen.size == np.unique(seen).size


# ----------------------------------------------------------------- routing
def check_route_bruteforce_all_eligible():
    """With capacity >= nb and p = K every eligible block is a candidate, so
    the route is the exact top-R of <qbar_j, kbar_i> over i <= j - L, which is
    found here from the full score matrix."""
    for (R, L, Hq, Hkv) in [(2, 1, 2, 1), (3, 2, 2, 2), (5, 1, 1, 1)]:
        p = _p(S=128, block=16, K=4, P=2, cap=8, probes=4, R=R, L=L, Hq=Hq, Hkv=Hkv, D=16)
        q = _rand((1, p.S, Hq, p.D), 15)
        k = _rand((1, p.S, Hkv, p.D), 16)
        cb = _unit_codebooks(2, 4, 8, 17)
        res = O.forward(q, k, k, cb, p, attention=False)
        g = Hq // Hkv
        for hq in range(Hq):
            sc = O.f32(O.f32(res.qbar[0, hq]) @ O.f32(res.kbar[0, hq // g]).T)
            for j in range(p.nb):
                elig = list(range(0, j - L + 1))
                best = sorted(sorted(elig, key=lambda i: (-sc[j, i], i))[:R])
                row = best + [-1] * (R - len(best)) + [i if i >= 0 else -1 for i in range(j - L + 1, j + 1)]
                assert list(res.sel[0, hq, j]) == row, (hq, j, list(res.sel[0, hq, j]), row)


def check_route_causal_and_fixed_slots():
    """No block is reachable from an earlier query block (Article, section
    "Monodratic Turns Sparse Attention Into a Retrieval Decision"), the
    locals are j-L+1..j, and every route has p**P x cap candidate slots
    (Report, Finite-range scaling: fixed candidate-slot checks)."""
    p = _p(S=256, block=16, K=4, P=2, cap=2, probes=2, R=3, L=2, D=16)
    q = _rand((2, p.S, 1, p.D), 18)
    k = _rand((2, p.S, 1, p.D), 19)
    cb = _unit_codebooks(2, 4, 8, 20)
    res = O.forward(q, k, k, cb, p, attention=False, keep_slots=True)
    for (b, h, j), slots in res.slots.items():
        assert slots.shape == (p.probes ** p.P, p.cap)
        sel = res.sel[b, h, j]
        remote, local = sel[: p.R], sel[p.R:]
        assert ((remote == -1) | ((remote >= 0) & (remote <= j - p.L))).all()
        assert list(local) == [i if i >= 0 else -1 for i in range(j - p.L + 1, j + 1)]
        v = remote[remote >= 0]
        assert np.array_equal(v, np.sort(v)) and set(v) <= set(slots[slots >= 0].tolist())
        assert (remote >= 0).sum() == min(p.R, res.ncand[b, h, j])


def check_eligibility_fixture():
    """Report, Learned sparse route: six blocks, one local block, five remote
    blocks eligible at the latest queries; two are selected."""
    with open(os.path.join(GOLDEN, "eligibility_six_blocks.json")) as f:
        g = json.load(f)
    p = _p(S=6 * 16, block=16, K=2, P=2, cap=6, probes=2, R=g["R"], L=g["L"], D=16)
    q = _rand((1, p.S, 1, p.D), 21)
    k = _rand((1, p.S, 1, p.D), 22)
    res = O.forward(q, k, k, _unit_codebooks(2, 2, 8, 23), p, attention=False)
    assert res.ncand[0, 0].tolist() == g["eligible_per_query_block"]
    assert int((res.sel[0, 0, 5, : p.R] >= 0).sum()) == g["selected_remote_at_last"]


# --------------------------------------------------------------- attention
def _sdpa(qr, kr, v, mask=None, causal=False, g=1):
    Q = torch.from_numpy(qr).permute(0, 2, 1, 3)
    Kt = torch.from_numpy(kr).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    V = torch.from_numpy(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(Q, Kt, V, attn_mask=m, is_causal=causal)
    return o.permute(0, 2, 1, 3).numpy()


def check_attention_dense_limit():
    """Capacity >= nb, p = K and R >= nb admit every earlier block, so the
    output is dense causal attention (PyTorch SDPA in float64 on the CPU).
    Also pins the 1/sqrt(D) scale and the query-head -> KV-head grouping."""
    for Hq, Hkv in [(1, 1), (4, 2)]:
        p = _p(S=64, block=16, K=2, P=2, cap=4, probes=2, R=4, L=1, Hq=Hq, Hkv=Hkv, D=16)
        q, k, v = _rand((1, p.S, Hq, p.D), 24), _rand((1, p.S, Hkv, p.D), 25), _rand((1, p.S, Hkv, p.D), 26)
        res = O.forward(q, k, v, _unit_codebooks(2, 2, 8, 27), p)
        ref = _sdpa(res.qr, res.kr, v, causal=True, g=Hq // Hkv)
        assert np.abs(res.out - ref).max() < 1e-12


def check_attention_local_only_is_block_diagonal():
    """R = 0, L = 1 (the local-only control): each block attends causally to
    itself only."""
    p = _p(S=64, block=16, R=0, L=1, D=16)
    q, k, v = _rand((1, p.S, 1, p.D), 28), _rand((1, p.S, 1, p.D), 29), _rand((1, p.S, 1, p.D), 30)
    res = O.forward(q, k, v, _unit_codebooks(2, 8, 8, 31), p)
    blk = np.arange(p.S) // p.block
    mask = (blk[:, None] == blk[None, :]) & np.tril(np.ones((p.S, p.S), dtype=bool))
    ref = _sdpa(res.qr, res.kr, v, mask=mask)
    assert np.abs(res.out - ref).max() < 1e-12


def check_attention_gather_equals_dense_mask():
    """The gathered selected-set softmax equals the dense masked softmax over
    the same selected positions (Report, Evidence: selected-mask oracle)."""
    p = _p(S=160, block=16, K=3, P=2, cap=2, probes=2, R=2, L=2, Hq=2, Hkv=1, D=16)
    q, k, v = _rand((2, p.S, 2, p.D), 32), _rand((2, p.S, 1, p.D), 33), _rand((2, p.S, 1, p.D), 34)
    res = O.forward(q, k, v, _unit_codebooks(2, 3, 8, 35), p)
    dense = O.attend_dense_mask(res.qr, res.kr, v, res.sel, p.block, p.softmax_scale)
    assert np.abs(res.out - dense).max() < 1e-12
    # and the selection is genuinely sparse here
    assert (res.sel[..., : p.R] >= 0).sum() < p.nb * p.R * 4


def check_softmax_lse_bruteforce():
    """The row normaliser against scipy's logsumexp of the dense score matrix
    under the selected-position mask; a query block with nothing selected is
    -inf; a row that sees only itself has the normaliser scale*<q'_t, k'_t>."""
    from scipy.special import logsumexp
    p = _p(S=96, block=16, K=3, P=2, cap=2, probes=2, R=2, L=1, Hq=2, Hkv=1, D=16)
    q, k, v = _rand((1, p.S, 2, p.D), 36), _rand((1, p.S, 1, p.D), 37), _rand((1, p.S, 1, p.D), 38)
    res = O.forward(q, k, v, _unit_codebooks(2, 3, 8, 39), p, attention=False)
    sel = res.sel.copy()
    sel[0, 1, 3] = -1                                   # nothing selected for (head 1, block 3)
    lse = O.softmax_lse(res.qr, res.kr, sel, p.block, p.softmax_scale)
    for hq in range(2):
        mask = O.selected_mask(sel[0, hq], p.S, p.block)
        sc = (res.qr[0, :, hq] @ res.kr[0, :, 0].T) * p.softmax_scale
        ref = logsumexp(np.where(mask, sc, -np.inf), axis=1)
        assert np.allclose(lse[0, hq], ref, rtol=0, atol=1e-12, equal_nan=False)
    assert np.isneginf(lse[0, 1, 3 * p.block:4 * p.block]).all()
    # local-only rows: token 0 of a block that selected only itself sees only itself
    own = O.softmax_lse(res.qr, res.kr, np.zeros_like(sel)[..., :1] + np.arange(p.nb)[None, None, :, None],
                        p.block, p.softmax_scale)
    t = 5 * p.block
    assert abs(own[0, 0, t] - p.softmax_scale * res.qr[0, t, 0] @ res.kr[0, t, 0]) < 1e-12


def check_backward_saved_output_identity():
    """The backward's row term rowsum(P * dP) equals <dout_t, out_t>: given
    attend()'s own output as the saved one, the gradients are unchanged."""
    p = _p(S=96, block=16, K=3, P=2, cap=2, probes=2, R=2, L=1, Hq=2, Hkv=1, D=16)
    q, k, v = _rand((1, p.S, 2, p.D), 40), _rand((1, p.S, 1, p.D), 41), _rand((1, p.S, 1, p.D), 42)
    res = O.forward(q, k, v, _unit_codebooks(2, 3, 8, 43), p)
    dout = _rand((1, p.S, 2, p.D), 44)
    a = O.attend_backward(res.qr, res.kr, v, res.sel, p.block, p.softmax_scale, dout)
    b = O.attend_backward(res.qr, res.kr, v, res.sel, p.block, p.softmax_scale, dout, saved_out=res.out)
    for x, y in zip(a, b):
        assert np.abs(x - y).max() < 1e-12
    # a perturbed saved output moves dq, dk but not dv
    c = O.attend_backward(res.qr, res.kr, v, res.sel, p.block, p.softmax_scale, dout, saved_out=res.out * 1.01)
    assert np.abs(c[2] - a[2]).max() < 1e-12 and np.abs(c[0] - a[0]).max() > 1e-6


# --------------------------------------------------------------- near ties
# A routing decision (a code, a probe set, a top-R set) is a near tie when the
# float32 gap at its boundary is below 1e-6*max(1,|s|), |s| the largest score
# magnitude among the items ranked; there either choice is correct.  These
# checks pin the margins, the scales and the threshold that decide which
# disagreements are excused: against a brute-force sorted() of scores
# computed exactly (rational arithmetic, then rounded to float32), planted
# exact ties, and gaps just on either side of the threshold.

def _f32_exact_dot(a, b) -> float:
    """<a, b> of two float32 vectors, summed exactly with rational
    arithmetic and rounded to float32: the score a float32 kernel aims at,
    whatever its summation order."""
    tot = sum(Fraction(float(x)) * Fraction(float(y))
              for x, y in zip(np.asarray(a, np.float32), np.asarray(b, np.float32)))
    return float(np.float32(float(tot)))


def _ranked(scores):
    """(score, index) pairs, best first (lower index first on equal scores)."""
    return [(-ns, i) for ns, i in sorted((-v, i) for i, v in enumerate(scores))]


def _close(x, y, ref):
    """Equal up to two float32 units in the last place at magnitude ref."""
    return abs(x - y) <= 2 * float(np.spacing(np.float32(max(abs(ref), 1e-30))))


def check_code_margin_bruteforce():
    """Key codes: the margin is the gap between the best and second-best
    score of the subspace, the scale its largest |score|; a key on a codeword
    that appears twice in the codebook is an exact tie (margin 0, a near tie)
    and goes to the lower index; K = 1 has no second choice (margin inf)."""
    P, K, d = 2, 6, 5
    cb = _unit_codebooks(P, K, d, 40)
    cb[1, 4] = cb[1, 2]                               # codewords 2 and 4 of subspace 1 are equal
    kbar = _rand((1, 2, 12, P * d), 41)
    kbar[0, 0, 0, d:] = 3.0 * cb[1, 2]                # exactly on the repeated codeword
    kbar[0, 1, 5, d:] = -0.25 * cb[1, 0] + 0.9 * cb[1, 4]
    addr, codes, margin = O.assign_codes(kbar, cb)
    scale = O.code_scale(kbar, cb)
    ties = 0
    for h, n, s in itertools.product(range(2), range(12), range(P)):
        sc = [_f32_exact_dot(kbar[0, h, n, s * d:(s + 1) * d], cb[s, k]) for k in range(K)]
        r = _ranked(sc)
        top = max(abs(v) for v in sc)
        assert codes[0, h, n, s] == r[0][1], (h, n, s)
        assert _close(margin[0, h, n, s], r[0][0] - r[1][0], top), (h, n, s, margin[0, h, n, s], r[:2])
        assert _close(scale[0, h, n, s], top, top), (h, n, s)
        if r[0][0] == r[1][0]:
            ties += 1
            assert margin[0, h, n, s] == 0 and O.near_tie(margin[0, h, n, s], scale[0, h, n, s])
    assert ties >= 2, "the planted exact ties must be seen"
    assert codes[0, 0, 0, 1] == 2, "an exact tie goes to the lower index"
    _, _, m1 = O.assign_codes(kbar, cb[:, :1])
    assert np.isinf(m1).all() and not O.near_tie(m1, 1.0).any()


def check_probe_margin_bruteforce():
    """Probes: the margin is the gap between ranks p and p+1 (the last probed
    codeword and the first left out); p = K probes everything (margin inf);
    with one probe and the best codeword repeated, the margin is exactly 0."""
    P, K, d = 2, 8, 6
    cb = _unit_codebooks(P, K, d, 42)
    qbar = _rand((1, 1, 25, P * d), 43)
    for p in (1, 3, 7):
        codes, margin = O.probe_codes(qbar, cb, p)
        for n, s in itertools.product(range(25), range(P)):
            sc = [_f32_exact_dot(qbar[0, 0, n, s * d:(s + 1) * d], cb[s, k]) for k in range(K)]
            r = _ranked(sc)
            assert list(codes[0, 0, n, s]) == [i for _, i in r[:p]]
            assert _close(margin[0, 0, n, s], r[p - 1][0] - r[p][0], max(abs(v) for v in sc)), (p, n, s)
    _, mK = O.probe_codes(qbar, cb, K)
    assert np.isinf(mK).all()
    cb2 = cb.copy()
    cb2[0, 6] = cb2[0, 1]
    q2 = np.concatenate([2.0 * cb2[0, 1], cb2[1, 0]]).astype(np.float64)[None, None, None, :]
    c2, m2 = O.probe_codes(q2, cb2, 1)
    assert c2[0, 0, 0, 0, 0] == 1 and m2[0, 0, 0, 0] == 0


def _score_rows(scores, D=8):
    """Query e_0 and one key summary per score: <q, k_i> = scores[i] exactly."""
    q = np.zeros(D)
    q[0] = 1.0
    k = np.zeros((len(scores), D))
    k[:, 0] = scores
    k[:, 1] = np.linspace(-3.0, 3.0, len(scores))     # orthogonal to q: no effect on the score
    return q, k


def check_route_margin_bruteforce():
    """Top-R: with every eligible block a candidate (capacity >= nb, p = K),
    the margin is the gap between ranks R and R+1 of the eligible scores, the
    scale their largest |score|, inf with at most R candidates or R = 0; a
    forced id leaves R-1 places, so the gap moves to ranks R-1 and R."""
    for (R, L, seed) in [(2, 1, 44), (3, 2, 45), (1, 1, 46)]:
        p = _p(S=192, block=16, K=4, P=2, cap=12, probes=4, R=R, L=L, D=16)
        q = _rand((1, p.S, 1, p.D), seed)
        k = _rand((1, p.S, 1, p.D), seed + 100)
        res = O.forward(q, k, k, _unit_codebooks(2, 4, 8, seed + 200), p, attention=False)
        for j in range(p.nb):
            elig = list(range(0, j - L + 1))
            sc = [_f32_exact_dot(res.qbar[0, 0, j], res.kbar[0, 0, i]) for i in elig]
            r = _ranked(sc)
            top = max((abs(v) for v in sc), default=0.0)
            m = res.sel_margin[0, 0, j]
            if len(elig) > R:
                assert _close(m, r[R - 1][0] - r[R][0], top), (R, j, m)
            else:
                assert np.isinf(m), (R, j, m)
            assert _close(res.sel_scale[0, 0, j], top, top), (R, j)
    # planted exact tie at the boundary: scores 0.5, 0.9, 0.7, 0.9, 0.1 with R = 1
    q, k = _score_rows([0.5, 0.9, 0.7, 0.9, 0.1])
    lists = np.array([[0, 1, 2, 3, 4, -1]])
    row = O.route_row(q, k, np.array([0]), lists, 6, 1, 1)
    assert row.sel[0] == 1 and row.margin == 0 and O.near_tie(row.margin, row.scale)
    assert row.scale == np.float32(0.9)
    row2 = O.route_row(q, k, np.array([0]), lists, 6, 2, 1)       # R = 2 takes both 0.9s
    assert list(row2.sel[:2]) == [1, 3] and _close(row2.margin, 0.9 - 0.7, 0.9)
    row0 = O.route_row(q, k, np.array([0]), lists, 6, 0, 1)
    assert np.isinf(row0.margin)
    rowf = O.route_row(q, k, np.array([0]), lists, 6, 2, 1, force=4)   # 4 forced, one place left
    assert list(rowf.sel[:2]) == [1, 4] and rowf.margin == 0


def check_near_tie_threshold():
    """The threshold is 1e-6*max(1,|s|): at |s| = 2 a gap of 16 float32 steps
    (1.91e-6) is a tie and 17 steps (2.03e-6) is not; at |s| = 0.5 the
    threshold is 1e-6, so 33 steps of 2^-25 (9.8e-7) are a tie and 34
    (1.01e-6) are not.  Codes and routes use the same rule."""
    d, P = 4, 2
    cb = np.zeros((P, 2 * d, d), dtype=np.float32)
    for s in range(P):
        for i in range(d):
            cb[s, 2 * i, i], cb[s, 2 * i + 1, i] = 1.0, -1.0
    for a, step, n_tie in [(2.0, 2.0 ** -23, 16), (0.5, 2.0 ** -25, 33)]:
        for n, expect in [(n_tie, True), (n_tie + 1, False)]:
            b = np.float32(a) - np.float32(n * step)
            kbar = np.zeros((1, 1, 1, P * d))
            kbar[0, 0, 0, :2] = [a, b]
            kbar[0, 0, 0, d] = 1.0
            _, codes, margin = O.assign_codes(kbar, cb)
            sc = O.code_scale(kbar, cb)
            assert codes[0, 0, 0, 0] == 0
            assert margin[0, 0, 0, 0] == np.float32(a) - b
            assert bool(O.near_tie(margin, sc)[0, 0, 0, 0]) == expect, (a, n)
            q, k = _score_rows([float(b), a, 0.25])
            row = O.route_row(q, k, np.array([0]), np.array([[0, 1, 2, -1]]), 3, 1, 1)
            assert row.sel[0] == 1 and bool(O.near_tie(row.margin, row.scale)) == expect, (a, n)


def check_decode_margins_bruteforce():
    """Decode: a token's probe margins and scales, and its top-R margin and
    scale over the completed blocks, equal a brute-force sort of its own
    rotated query's scores."""
    p = _p(S=128, block=16, K=4, P=2, cap=8, probes=2, R=2, L=1, D=16)
    B = 2
    q, k, v = _rand((B, p.S, 1, p.D), 47), _rand((B, p.S, 1, p.D), 48), _rand((B, p.S, 1, p.D), 49)
    cb = _unit_codebooks(2, 4, 8, 50)
    st = O.decode_init(p, B)
    dsub = p.D // p.P
    for t in range(p.S):
        o = O.decode_step(st, q[:, t], k[:, t], v[:, t], cb, p)
        if t % 7:
            continue
        qr = O.rope_at(q[:, t], t, p.rope_base)
        j = t // p.block
        for b in range(B):
            for s in range(p.P):
                sc = [_f32_exact_dot(qr[b, 0, s * dsub:(s + 1) * dsub], cb[s, kk]) for kk in range(p.K)]
                r = _ranked(sc)
                top = max(abs(x) for x in sc)
                assert _close(o.qcode_margin[b, 0, s], r[p.probes - 1][0] - r[p.probes][0], top), (t, b, s)
                assert _close(o.qcode_scale[b, 0, s], top, top)
            pa = O.probe_addresses(o.qcodes[b, 0], p.K)
            cand = sorted(i for i in st.lists[b, 0, pa].ravel() if 0 <= i <= j - p.L)
            sc = [_f32_exact_dot(qr[b, 0], st.kbar[b, 0, i]) for i in cand]
            r = _ranked(sc)
            top = max((abs(x) for x in sc), default=0.0)
            assert _close(o.sel_scale[b, 0], top, top), (t, b)
            if len(cand) > p.R:
                assert _close(o.sel_margin[b, 0], r[p.R - 1][0] - r[p.R][0], top), (t, b)
            else:
                assert np.isinf(o.sel_margin[b, 0])


ALL_CHECKS = [v for k, v in sorted(globals().items()) if k.startswith("check_")]
