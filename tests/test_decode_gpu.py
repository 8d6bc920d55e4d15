"""GPU parity of the decode path (mdr_decode_prefill + mdr_decode_step, one
token at a time with an incremental index) against the oracle's decode
(oracle.mdr_oracle.decode_step) on the same seeded inputs.

The bar is the one stated in tests/parity_util.py: selected blocks,
candidate counts and addresses bit-exact unless the oracle flags the deciding
float32 margin as a near tie (then the GPU's choice must be a valid one, and
the oracle continues from it); lists and loads bit-exact; summaries within
1e-5; attention outputs of every token within 1e-5 (float32) or 2e-2
row-relative (bf16), over the GPU's selection."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import parity_util as U
from workloads import AR, CAPACITY, TINY, SCALING_32K, make_inputs

pytestmark = pytest.mark.gpu


def _gpu_decode(w, inp, S0, t_end):
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    q, k, v, cb = U.to_device(inp, w)
    st = mdr.DecodeState.empty(cfg)
    ws = mdr.decode_workspace(cfg)
    mdr.mdr_decode_prefill(cfg, S0, k[:, :S0].contiguous(), v[:, :S0].contiguous(), cb, st, ws)
    out_t = torch.empty(w.B, w.Hq, w.D, dtype=q.dtype, device=q.device)
    sel_t = torch.empty(w.B, w.Hq, w.R + w.L, dtype=torch.int32, device=q.device)
    nc_t = torch.empty(w.B, w.Hq, dtype=torch.int32, device=q.device)
    steps = []
    for t in range(S0, t_end):
        mdr.mdr_decode_step(cfg, t, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), cb, st,
                            out_t, sel_t, ws, ncand_t=nc_t)
        steps.append((out_t.float().cpu().numpy(), sel_t.cpu().numpy(), nc_t.cpu().numpy()))
    assert mdr.mdr_read_device_status(ws) == 0
    state = {f: getattr(st.idx, f).cpu().numpy() for f in ("kbar", "addr", "lists", "load", "overflow", "maxload")}
    return steps, state


def _check_key(w, codes, margin, scale, kbar, g_addr, codebooks):
    """The GPU's addresses of completed blocks [..]: the oracle's codes, or,
    where the oracle's margin is a near tie, a codeword within the threshold
    of the best.  Returns the number of blocks taken the other way."""
    K, P = w.K, w.P
    g_codes = (g_addr[..., None] // (K ** np.arange(P - 1, -1, -1))) % K
    diff = g_codes != codes
    tie = O.near_tie(margin, scale)
    assert not (diff & ~tie).any(), f"{int((diff & ~tie).sum())} key codes differ outside near ties"
    sc = O.codeword_scores(kbar, codebooks)
    g_sc = np.take_along_axis(sc, g_codes[..., None], axis=-1)[..., 0]
    assert (sc.max(axis=-1) - g_sc < O.TIE_REL * np.maximum(1.0, scale))[diff].all()
    return int(diff.any(axis=-1).sum())


def _check_step(w, r, st, t, g_out, g_sel, g_nc):
    """One token: the GPU's routes equal the oracle's outside near ties (and
    stay causal and listed inside one); candidate counts equal unless the
    probes are a near tie; the attention of every (sequence, head) equals the
    oracle's over the GPU's selection.  Returns the routes taken the other
    way."""
    j = t // w.block
    g = w.Hq // w.Hkv
    loc = [i if i >= 0 else -1 for i in range(j - w.L + 1, j + 1)]
    n = 0
    for b in range(w.B):
        for hq in range(w.Hq):
            qtie = bool(O.near_tie(r.qcode_margin[b, hq], r.qcode_scale[b, hq]).any())
            stie = bool(O.near_tie(r.sel_margin[b, hq], r.sel_scale[b, hq]))
            rem = g_sel[b, hq, : w.R]
            assert ((rem == -1) | ((rem >= 0) & (rem <= j - w.L))).all(), (t, b, hq, g_sel[b, hq])
            assert list(g_sel[b, hq, w.R:]) == loc
            if not np.array_equal(g_sel[b, hq], r.sel[b, hq]):
                assert qtie or stie, (t, b, hq, g_sel[b, hq], r.sel[b, hq])
                listed = set(st.lists[b, hq // g].ravel().tolist())
                assert set(rem[rem >= 0].tolist()) <= listed, (t, b, hq)
                n += 1
            if not qtie:
                assert g_nc[b, hq] == r.ncand[b, hq], (t, b, hq)
            ref = r.out[b, hq]
            if w.dtype == "f32":
                assert np.abs(g_out[b, hq] - ref).max() <= U.TOL_F32_OUT, (t, b, hq)
            else:
                assert np.linalg.norm(g_out[b, hq] - ref) <= U.TOL_BF16_REL * np.linalg.norm(ref), (t, b, hq)
    return n


def _compare(w, inp, S0, t_end, max_ties=2):
    """Decode tokens S0..t_end-1 on the GPU after a prefill of S0 tokens and
    step the oracle through every token in lock step: a block's address and
    a token's selection are the GPU's where they differ inside a near tie, so
    everything after them (lists, later routes, every token's attention) is
    compared against the oracle re-run with the GPU's choice."""
    g_steps, g_state = _gpu_decode(w, inp, S0, t_end)
    p = O.Params.of(w)
    st = O.decode_init(p, w.B)
    ties = 0
    for t in range(t_end):
        done = (t + 1) % w.block == 0
        jd = t // w.block
        g_addr = g_state["addr"][:, :, jd] if done else None
        gs = g_steps[t - S0] if t >= S0 else None
        r = O.decode_step(st, inp.q[:, t], inp.k[:, t], inp.v[:, t], inp.codebooks, p,
                          addr=g_addr, sel=None if gs is None else gs[1])
        if done:
            ties += _check_key(w, r.key_codes, r.key_margin, r.key_scale, st.kbar[:, :, jd], g_addr,
                               inp.codebooks)
        if gs is not None:
            ties += _check_step(w, r, st, t, *gs)
    nbd = t_end // w.block                                  # completed blocks
    np.testing.assert_allclose(g_state["kbar"][:, :, :nbd], st.kbar[:, :, :nbd], rtol=1e-5, atol=1e-5)
    assert np.array_equal(g_state["addr"][:, :, :nbd], st.addr[:, :, :nbd])
    assert np.array_equal(g_state["lists"], st.lists)
    assert np.array_equal(g_state["load"], st.load)
    assert np.array_equal(g_state["overflow"], st.overflow) and np.array_equal(g_state["maxload"], st.maxload)
    assert ties <= max_ties, ties
    print(f"decode ties {w.name}: {ties}")
    return ties


def test_decode_from_empty_f32():
    """Every token of the tiny float32 case decoded from an empty state: six
    blocks complete on the way."""
    inp = make_inputs(TINY, 0)
    _compare(TINY, inp, 0, TINY.S)


def test_decode_after_prefill_bf16():
    """Planted-block workload: prefill four blocks, decode two more (both
    complete during decoding), two sequences."""
    w = AR.with_(B=2)
    inp = make_inputs(w, 1)
    _compare(w, inp, 256, w.S)


def test_decode_gqa_overflow_bf16():
    """Grouped query heads (3 per KV head) and tiny lists (capacity 1):
    appends overflow and the route sees only the first block of each
    address."""
    w = CAPACITY.with_(S=1024, Hq=6, Hkv=2, cap=1, K=4, probes=2, R=4, L=2, keys="gaussian")
    inp = make_inputs(w, 2)
    _compare(w, inp, 512, 768)


def test_decode_local_only_f32():
    """R = 0: the route keeps only the local blocks."""
    w = TINY.with_(R=0, L=2)
    inp = make_inputs(w, 3)
    _compare(w, inp, 32, w.S)


def test_decode_many_candidates_bf16():
    """Four codewords per subspace (16 addresses) probed four deep: every
    list is probed, so a token sees every eligible block as a candidate
    (more than 32): the route takes its best R by rounds of arg-max rather
    than by the one-pass ranking used for at most 32."""
    w = AR.with_(B=1, S=4096, K=4, probes=4, cap=16, R=8, L=2, keys="gaussian")
    inp = make_inputs(w, 8)
    _compare(w, inp, 3072, 3072 + 66)


def test_decode_block128_gqa_bf16():
    """Blocks of 128 tokens at D = 128 with four query heads per KV head (the
    long workload's head shape, shortened): a selected block is read in two
    passes of 64 rows, so the running maximum is rescaled between passes; a
    block completes during decoding."""
    from workloads import LONG
    w = LONG.with_(S=2048, Hq=8, Hkv=2, keys="gaussian")
    inp = make_inputs(w, 6)
    _compare(w, inp, 1536, 1536 + 129)


@pytest.mark.parametrize("D,block,S", [(64, 32, 192), (128, 64, 384)])
def test_decode_f32_wide_rows(D, block, S):
    """float32 rows of 64 and 128 coordinates (16 and 32 lanes per row; at
    D = 128 a block of 64 rows takes two passes)."""
    w = TINY.with_(D=D, block=block, S=S)
    inp = make_inputs(w, 7)
    _compare(w, inp, S // 2, S)


def test_prefill_state_equals_oracle_index():
    """mdr_decode_prefill of a prefix holds the oracle's index of that prefix
    (the batch build), in the state's own strides (capacity larger than the
    prefix, two sequences)."""
    import torch
    from learned_product_hash_b200 import mdr
    w = AR.with_(B=2)
    inp = make_inputs(w, 4)
    S0 = 192
    cfg = mdr.make_config(w)
    q, k, v, cb = U.to_device(inp, w)
    st = mdr.DecodeState.empty(cfg)
    ws = mdr.decode_workspace(cfg)
    mdr.mdr_decode_prefill(cfg, S0, k[:, :S0].contiguous(), v[:, :S0].contiguous(), cb, st, ws)
    torch.cuda.synchronize()
    p = O.Params.of(w.with_(S=S0))
    kr = O.rope(inp.k[:, :S0].astype(np.float64), p.rope_base)
    kbar, addr, _, _, lists, load, overflow, maxload = O.build_index(kr, inp.codebooks, p)
    nb0 = S0 // w.block
    np.testing.assert_allclose(st.idx.kbar.cpu().numpy()[:, :, :nb0], kbar, rtol=1e-5, atol=1e-5)
    assert np.array_equal(st.idx.addr.cpu().numpy()[:, :, :nb0], addr)
    assert np.array_equal(st.idx.lists.cpu().numpy(), lists)
    assert np.array_equal(st.idx.load.cpu().numpy(), load)
    assert np.array_equal(st.idx.overflow.cpu().numpy(), overflow)
    g_kr = st.krot.float().cpu().numpy()[:, :S0]
    rel = np.abs(g_kr - kr).max() / np.abs(kr).max()
    assert rel <= 1e-2                                   # bf16 rounding of the rotated keys
    assert np.array_equal(st.v.float().cpu().numpy()[:, :S0], inp.v[:, :S0])


def test_decode_full_size_last_block():
    """The 32K workload: prefill 511 blocks, decode the last 64 tokens (the
    last block completes at the final step).  The oracle's state is the
    batch build of the prefix (on the GPU's addresses where they differ
    inside a near tie), then its own decode steps in lock step with the GPU's;
    every eighth step and the last are compared."""
    w = SCALING_32K
    inp = make_inputs(w, 5)
    S0 = w.S - w.block
    nb0 = S0 // w.block
    g_steps, g_state = _gpu_decode(w, inp, S0, w.S)
    p = O.Params.of(w)
    st = O.decode_init(p, w.B)
    kr = O.rope(inp.k[:, :S0].astype(np.float64), p.rope_base)
    pp = O.Params.of(w.with_(S=S0))
    g_addr0 = g_state["addr"][:, :, :nb0]
    kbar, _, codes, margin, lists, load, _, _ = O.build_index(kr, inp.codebooks, pp, addr=g_addr0)
    ties = _check_key(w, codes, margin, O.code_scale(kbar, inp.codebooks), kbar, g_addr0, inp.codebooks)
    st.kr[:, :S0] = kr
    st.v[:, :S0] = inp.v[:, :S0]
    st.kbar[:, :, :nb0] = kbar
    st.addr[:, :, :nb0] = g_addr0
    st.lists[:], st.load[:] = lists, load
    st.t = S0
    for i, t in enumerate(range(S0, w.S)):
        g_out, g_sel, g_nc = g_steps[i]
        done = t == w.S - 1
        g_addr = g_state["addr"][:, :, w.nb - 1] if done else None
        r = O.decode_step(st, inp.q[:, t], inp.k[:, t], inp.v[:, t], inp.codebooks, p, addr=g_addr, sel=g_sel)
        if done:
            ties += _check_key(w, r.key_codes, r.key_margin, r.key_scale, st.kbar[:, :, w.nb - 1], g_addr,
                               inp.codebooks)
        if i % 8 and not done:
            continue
        ties += _check_step(w, r, st, t, g_out, g_sel, g_nc)
    assert np.array_equal(g_state["load"], st.load)
    assert np.array_equal(g_state["lists"], st.lists)
    assert ties <= U.full_size_tie_budget(w), ties
    print(f"decode ties {w.name}: {ties}")
