"""GPU parity of the decode path (mdr_decode_prefill + mdr_decode_step, one
token at a time with an incremental index) against the oracle's decode
(oracle.mdr_oracle.decode_step) on the same seeded inputs.

The bar is the one stated in tests/parity_util.py: probed codewords, selected
blocks, candidate counts, addresses, lists and loads bit-exact unless the
oracle flags the deciding float32 margin as a near tie; summaries within
1e-5; attention outputs within 1e-5 (float32) or 2e-2 row-relative (bf16)."""
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


def _oracle_decode(w, inp, S0, t_end):
    p = O.Params.of(w)
    st = O.decode_init(p, w.B)
    steps = []
    for t in range(t_end):
        o = O.decode_step(st, inp.q[:, t], inp.k[:, t], inp.v[:, t], inp.codebooks, p)
        if t >= S0:
            steps.append(o)
    return steps, st


def _compare(w, inp, S0, t_end):
    g_steps, g_state = _gpu_decode(w, inp, S0, t_end)
    r_steps, r_state = _oracle_decode(w, inp, S0, t_end)
    nbd = t_end // w.block                                  # completed blocks
    g = w.Hq // w.Hkv
    # Key side: blocks whose code decision is a near tie may differ; the
    # (sequence, KV head) holding one is compared for validity only.
    _, _, kmargin = O.assign_codes(r_state.kbar[:, :, :nbd], inp.codebooks)
    sc = O.codeword_scores(r_state.kbar[:, :, :nbd], inp.codebooks).max(axis=-1)
    key_tie = O.near_tie(kmargin, sc).any(axis=(-1, -2))    # [B, Hkv]
    np.testing.assert_allclose(g_state["kbar"][:, :, :nbd], r_state.kbar[:, :, :nbd], rtol=1e-5, atol=1e-5)
    for b in range(w.B):
        for h in range(w.Hkv):
            if key_tie[b, h]:
                continue
            assert np.array_equal(g_state["addr"][b, h, :nbd], r_state.addr[b, h, :nbd]), (b, h)
            assert np.array_equal(g_state["lists"][b, h], r_state.lists[b, h]), (b, h)
            assert np.array_equal(g_state["load"][b, h], r_state.load[b, h]), (b, h)
            assert g_state["overflow"][b, h] == r_state.overflow[b, h]
            assert g_state["maxload"][b, h] == r_state.maxload[b, h]
    checked = 0
    for (g_out, g_sel, g_nc), r in zip(g_steps, r_steps):
        for b in range(w.B):
            for hq in range(w.Hq):
                if key_tie[b, hq // g]:
                    continue
                tie = O.near_tie(r.qcode_margin[b, hq], r.qcode_scale[b, hq]).any() or \
                    O.near_tie(r.sel_margin[b, hq], r.sel_scale[b, hq])
                if tie:
                    continue
                assert np.array_equal(g_sel[b, hq], r.sel[b, hq]), (b, hq, g_sel[b, hq], r.sel[b, hq])
                assert g_nc[b, hq] == r.ncand[b, hq]
                ref = r.out[b, hq]
                if w.dtype == "f32":
                    assert np.abs(g_out[b, hq] - ref).max() <= U.TOL_F32_OUT
                else:
                    assert np.linalg.norm(g_out[b, hq] - ref) <= U.TOL_BF16_REL * np.linalg.norm(ref)
                checked += 1
    assert checked >= 0.9 * len(g_steps) * w.B * w.Hq
    return checked


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
    last block completes at the final step); a sample of steps is compared
    with the oracle, whose state is the batch build of the prefix followed by
    its own decode steps."""
    import torch
    from learned_product_hash_b200 import mdr
    w = SCALING_32K
    inp = make_inputs(w, 5)
    S0 = w.S - w.block
    g_steps, g_state = _gpu_decode(w, inp, S0, w.S)
    p = O.Params.of(w)
    st = O.decode_init(p, w.B)
    kr = O.rope(inp.k[:, :S0].astype(np.float64), p.rope_base)
    pp = O.Params.of(w.with_(S=S0))
    kbar, addr, _, _, lists, load, _, _ = O.build_index(kr, inp.codebooks, pp)
    st.kr[:, :S0] = kr
    st.v[:, :S0] = inp.v[:, :S0]
    st.kbar[:, :, : S0 // w.block] = kbar
    st.addr[:, :, : S0 // w.block] = addr
    st.lists[:], st.load[:] = lists, load
    st.t = S0
    for i, t in enumerate(range(S0, w.S)):
        r = O.decode_step(st, inp.q[:, t], inp.k[:, t], inp.v[:, t], inp.codebooks, p)
        if i % 8 and t != w.S - 1:
            continue
        g_out, g_sel, g_nc = g_steps[i]
        for hq in range(w.Hq):
            if O.near_tie(r.qcode_margin[0, hq], r.qcode_scale[0, hq]).any():
                continue
            if O.near_tie(r.sel_margin[0, hq], r.sel_scale[0, hq]):
                continue
            assert np.array_equal(g_sel[0, hq], r.sel[0, hq]), (t, hq)
            assert np.linalg.norm(g_out[0, hq] - r.out[0, hq]) <= U.TOL_BF16_REL * np.linalg.norm(r.out[0, hq])
    nb = w.nb
    assert np.array_equal(g_state["load"], st.load)
    assert np.array_equal(g_state["addr"][:, :, nb - 1], st.addr[:, :, nb - 1])
