"""The oracle's decode path (one token at a time, incremental index) against
the batch build and against closed-form attention (no GPU)."""
import numpy as np
import pytest

from oracle import mdr_oracle as O


def _p(**kw):
    base = dict(B=1, S=96, Hq=2, Hkv=1, D=32, block=16, P=2, K=4, cap=8,
                probes=2, R=2, L=1, rope_base=10000.0, scale=0.0)
    base.update(kw)
    return O.Params(**base)


def _inputs(p, B, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, p.S, p.Hq, p.D))
    k = rng.standard_normal((B, p.S, p.Hkv, p.D))
    v = rng.standard_normal((B, p.S, p.Hkv, p.D))
    c = rng.standard_normal((p.P, p.K, p.D // p.P))
    c = (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)
    return q, k, v, c


def _decode_all(p, q, k, v, c):
    st = O.decode_init(p, q.shape[0])
    outs = [O.decode_step(st, q[:, t], k[:, t], v[:, t], c, p) for t in range(p.S)]
    return st, outs


@pytest.mark.parametrize("cap", [1, 3, 8])
def test_incremental_index_equals_batch_build(cap):
    """Appending blocks as they complete gives the index the batch build
    gives for the same keys: summaries, addresses, lists (first cap per
    address, ascending), loads, overflow and maximum load."""
    p = _p(cap=cap, K=2)
    q, k, v, c = _inputs(p, 2, 1)
    st, _ = _decode_all(p, q, k, v, c)
    kr = O.rope(k, p.rope_base)
    kbar, addr, _, _, lists, load, overflow, maxload = O.build_index(kr, c, p)
    np.testing.assert_allclose(st.kr, kr, rtol=0, atol=1e-12)
    np.testing.assert_allclose(st.kbar, kbar, rtol=0, atol=1e-12)
    assert np.array_equal(st.addr, addr)
    assert np.array_equal(st.lists, lists)
    assert np.array_equal(st.load, load)
    assert np.array_equal(st.overflow, overflow)
    assert np.array_equal(st.maxload, maxload)


def test_index_before_a_block_completes():
    """A block is not in the index until its last token has arrived."""
    p = _p()
    q, k, v, c = _inputs(p, 1, 2)
    st = O.decode_init(p, 1)
    for t in range(p.block - 1):
        O.decode_step(st, q[:, t], k[:, t], v[:, t], c, p)
    assert st.load.sum() == 0 and (st.addr == -1).all()
    O.decode_step(st, q[:, p.block - 1], k[:, p.block - 1], v[:, p.block - 1], c, p)
    assert st.load.sum() == p.Hkv and (st.addr[:, :, 0] >= 0).all() and (st.addr[:, :, 1:] == -1).all()


def _dense_causal(qr_t, kr, v, t, scale):
    """softmax over every s <= t of scale * <q'_t, k'_s>, applied to v_s,
    written out directly."""
    s = np.array([scale * float(np.dot(qr_t, kr[u])) for u in range(t + 1)])
    w = np.exp(s - s.max())
    return (w[:, None] * v[: t + 1]).sum(axis=0) / w.sum()


def test_dense_limit_is_full_causal_attention():
    """Every address probed (p = K), every block stored (cap >= nb) and R >=
    nb: each token attends to every earlier token -- dense causal attention."""
    p = _p(K=2, probes=2, cap=8, R=6, L=1, Hq=2, Hkv=2)
    q, k, v, c = _inputs(p, 1, 3)
    st, outs = _decode_all(p, q, k, v, c)
    for t in (0, 5, 15, 16, 40, 95):
        for h in range(p.Hq):
            qr_t = O.rope_at(q[0, t, h], t, p.rope_base)
            ref = _dense_causal(qr_t, st.kr[0, :, h], st.v[0, :, h], t, p.softmax_scale)
            np.testing.assert_allclose(outs[t].out[0, h], ref, rtol=0, atol=1e-12)


def test_local_only_is_sliding_block_window():
    """R = 0: token t of block j attends to the tokens of blocks j-L+1..j up
    to itself."""
    p = _p(R=0, L=2)
    q, k, v, c = _inputs(p, 1, 4)
    st, outs = _decode_all(p, q, k, v, c)
    for t in (0, 17, 31, 32, 70, 95):
        j = t // p.block
        lo = max(0, (j - p.L + 1) * p.block)
        for h in range(p.Hq):
            qr_t = O.rope_at(q[0, t, h], t, p.rope_base)
            s = np.array([p.softmax_scale * float(np.dot(qr_t, st.kr[0, u, 0])) for u in range(lo, t + 1)])
            w = np.exp(s - s.max())
            ref = (w[:, None] * st.v[0, lo:t + 1, 0]).sum(axis=0) / w.sum()
            np.testing.assert_allclose(outs[t].out[0, h], ref, rtol=0, atol=1e-12)
            assert list(outs[t].sel[0, h]) == [b if b >= 0 else -1 for b in range(j - p.L + 1, j + 1)]


def test_route_uses_the_tokens_own_query_and_only_earlier_blocks():
    """The decode route of token t is the batch route_row with the token's
    rotated query as the query summary; no selected remote block is later
    than j - L, and every remote one is in the probed lists."""
    p = _p(K=4, probes=2, cap=2, R=2, L=1)
    q, k, v, c = _inputs(p, 1, 5)
    st = O.decode_init(p, 1)
    for t in range(p.S):
        o = O.decode_step(st, q[:, t], k[:, t], v[:, t], c, p)
        j = t // p.block
        remote = o.sel[0, :, : p.R]
        assert (remote[remote >= 0] <= j - p.L).all()
        for h in range(p.Hq):
            qr_t = O.rope_at(q[0, t, h], t, p.rope_base)
            sc = O.codeword_scores(qr_t, c)
            for s in range(p.P):       # brute-force top-p per subspace
                order = sorted(range(p.K), key=lambda kk: (-sc[s, kk], kk))[: p.probes]
                assert list(o.qcodes[0, h, s]) == order
            pa = O.probe_addresses(o.qcodes[0, h], p.K)
            listed = set(st.lists[0, 0][pa].ravel()) - {-1}
            assert set(remote[h][remote[h] >= 0]) <= listed
