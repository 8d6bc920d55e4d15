"""The oracle's backward (gradients of the mixer's output with the route held
fixed) pinned without a GPU: central finite differences of the forward on
every input coordinate, autograd of PyTorch's scaled_dot_product_attention
in the dense and local-only limits, and planted mistakes."""
import numpy as np
import pytest
import torch

from oracle import mdr_oracle as O


def _p(**kw):
    base = dict(B=1, S=32, Hq=2, Hkv=1, D=8, block=8, P=2, K=2, cap=4, probes=1, R=1, L=1,
                rope_base=100.0, scale=0.0)
    base.update(kw)
    return O.Params(**base)


def _inputs(p, seed):
    r = np.random.default_rng(seed)
    q = r.standard_normal((p.B, p.S, p.Hq, p.D))
    k = r.standard_normal((p.B, p.S, p.Hkv, p.D))
    v = r.standard_normal((p.B, p.S, p.Hkv, p.D))
    c = r.standard_normal((p.P, p.K, p.D // p.P))
    c = (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)
    G = r.standard_normal((p.B, p.S, p.Hq, p.D))
    return q, k, v, c, G


def check_gradients_equal_finite_differences():
    """dL/dq, dL/dk, dL/dv of L = sum(out * G) with the route fixed, against
    central differences (h = 1e-5) on every coordinate of q, k and v; two
    query heads share the KV head, so the key and value gradients add over
    the group."""
    p = _p()
    q, k, v, c, G = _inputs(p, 1)
    dq, dk, dv, sel = O.backward(q, k, v, c, p, G)
    assert (sel[..., : p.R] >= 0).any()                  # some remote blocks are attended

    def loss(q_, k_, v_):
        out = O.attend(O.rope(q_, p.rope_base), O.rope(k_, p.rope_base), v_, sel, p.block, p.softmax_scale)
        return float((out * G).sum())

    h = 1e-5
    for name, x, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.empty_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            args_m = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, fd, rtol=0, atol=2e-7, err_msg=name)


def _sdpa_grads(qr, kr, v, G, scale, mask=None):
    """Autograd of torch's SDPA (float64, CPU) on the rotated q', k'; the KV
    head is repeated for its query heads, so its gradient adds over them."""
    g = qr.shape[2] // kr.shape[2]
    Q = torch.tensor(qr.transpose(0, 2, 1, 3), requires_grad=True)
    K = torch.tensor(kr.transpose(0, 2, 1, 3), requires_grad=True)
    V = torch.tensor(v.transpose(0, 2, 1, 3), requires_grad=True)
    Ke, Ve = K.repeat_interleave(g, dim=1), V.repeat_interleave(g, dim=1)
    if mask is None:
        out = torch.nn.functional.scaled_dot_product_attention(Q, Ke, Ve, is_causal=True, scale=scale)
    else:
        out = torch.nn.functional.scaled_dot_product_attention(Q, Ke, Ve, attn_mask=torch.tensor(mask), scale=scale)
    (out * torch.tensor(G.transpose(0, 2, 1, 3))).sum().backward()
    return (Q.grad.numpy().transpose(0, 2, 1, 3), K.grad.numpy().transpose(0, 2, 1, 3),
            V.grad.numpy().transpose(0, 2, 1, 3))


def check_dense_limit_equals_sdpa_autograd():
    """Every block selected (p = K, cap >= nb, R >= nb): the attention is
    dense causal attention, and its gradients are autograd's."""
    p = _p(S=64, Hq=4, Hkv=2, D=16, K=2, probes=2, cap=8, R=8, L=1)
    q, k, v, c, G = _inputs(p, 2)
    sel = O.forward(q, k, v, c, p, attention=False).sel
    qr, kr = O.rope(q, p.rope_base), O.rope(k, p.rope_base)
    dq, dk, dv = O.attend_backward(qr, kr, v, sel, p.block, p.softmax_scale, G)
    rq, rk, rv = _sdpa_grads(qr, kr, v, G, p.softmax_scale)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def check_local_only_equals_block_diagonal_sdpa_autograd():
    """R = 0, L = 1: each block attends causally to itself only."""
    p = _p(S=48, Hq=2, Hkv=2, D=16, R=0, L=1)
    q, k, v, c, G = _inputs(p, 3)
    sel = O.forward(q, k, v, c, p, attention=False).sel
    qr, kr = O.rope(q, p.rope_base), O.rope(k, p.rope_base)
    dq, dk, dv = O.attend_backward(qr, kr, v, sel, p.block, p.softmax_scale, G)
    blk = np.arange(p.S) // p.block
    mask = (blk[:, None] == blk[None, :]) & np.tril(np.ones((p.S, p.S), dtype=bool))
    rq, rk, rv = _sdpa_grads(qr, kr, v, G, p.softmax_scale, mask)
    for a, b in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def check_rows_without_selection_get_zero_gradients():
    """A caller-made selection with an empty row: its queries get zero dq and
    contribute nothing to dk, dv."""
    p = _p()
    q, k, v, c, G = _inputs(p, 4)
    sel = O.forward(q, k, v, c, p, attention=False).sel.copy()
    qr, kr = O.rope(q, p.rope_base), O.rope(k, p.rope_base)
    base = O.attend_backward(qr, kr, v, sel, p.block, p.softmax_scale, G)
    sel[0, 1, 2] = -1
    G2 = G.copy()
    G2[0, 2 * p.block:3 * p.block, 1] = 0.0              # that row's upstream gradient no longer matters
    dq, dk, dv = O.attend_backward(qr, kr, v, sel, p.block, p.softmax_scale, G)
    assert (dq[0, 2 * p.block:3 * p.block, 1] == 0).all()
    sel_b = O.forward(q, k, v, c, p, attention=False).sel
    ref = O.attend_backward(qr, kr, v, sel_b, p.block, p.softmax_scale, G2)
    np.testing.assert_allclose(dk, ref[1], atol=1e-12)
    np.testing.assert_allclose(dv, ref[2], atol=1e-12)
    assert not np.allclose(base[1], dk)


CHECKS = [check_gradients_equal_finite_differences, check_dense_limit_equals_sdpa_autograd,
          check_local_only_equals_block_diagonal_sdpa_autograd, check_rows_without_selection_get_zero_gradients]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_backward_pin(check):
    check()


# ------------------------------------------------ planted mistakes are caught
_BWD = O.attend_backward


def _mutant(kind):
    def attend_backward(qr, kr, v, sel, bs, scale, dout):
        B, S, Hq, D = qr.shape
        g = Hq // kr.shape[2]
        dq, dk, dv = np.zeros_like(qr), np.zeros_like(kr), np.zeros_like(v)
        for b in range(B):
            for hq in range(Hq):
                h = hq % kr.shape[2] if kind == "wrong_kv_head" else hq // g
                for j in range(S // bs):
                    toks = O.selected_tokens(sel[b, hq, j], bs)
                    if toks.size == 0:
                        continue
                    qpos = np.arange(j * bs, (j + 1) * bs)
                    Q, Kt, Vt = qr[b, qpos, hq], kr[b, toks, h], v[b, toks, h]
                    s = (Q @ Kt.T) * scale
                    if kind != "no_causal_mask":
                        s[toks[None, :] > qpos[:, None]] = -np.inf
                    P = np.exp(s - s.max(axis=1, keepdims=True))
                    P /= P.sum(axis=1, keepdims=True)
                    dO = dout[b, qpos, hq]
                    dv[b, toks, h] += P.T @ dO
                    dP = dO @ Vt.T
                    dS = P * dP if kind == "no_row_term" else P * (dP - (P * dP).sum(axis=1, keepdims=True))
                    sc = 1.0 if kind == "no_scale" else scale
                    dq[b, qpos, hq] = sc * dS @ Kt
                    if kind == "dk_overwritten":
                        dk[b, toks, h] = sc * dS.T @ Q
                    else:
                        dk[b, toks, h] += sc * dS.T @ Q
        return dq, dk, dv
    return attend_backward


def _rope_transpose_wrong_sign(y, base):
    B, S, H, D = y.shape
    th = O.rope_angles(S, D, base).astype(np.float64)
    c, s = np.cos(th)[None, :, None, :], np.sin(th)[None, :, None, :]
    y1, y2 = y[..., : D // 2], y[..., D // 2:]
    return np.concatenate([y1 * c - y2 * s, y2 * c + y1 * s], axis=-1)


@pytest.mark.parametrize("attr,fn", [("attend_backward", _mutant(k)) for k in
                                     ("no_row_term", "no_causal_mask", "no_scale", "dk_overwritten", "wrong_kv_head")] +
                         [("rope_transpose", _rope_transpose_wrong_sign)],
                         ids=["no_row_term", "no_causal_mask", "no_scale", "dk_overwritten", "wrong_kv_head",
                              "rope_transpose_wrong_sign"])
def test_backward_mutation_is_caught(attr, fn, monkeypatch):
    monkeypatch.setattr(O, attr, fn)
    caught = 0
    for check in CHECKS:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no backward check catches {fn.__name__}"
