"""Plant a plausible mistake in the CPU oracle and require that at least one
pin check catches it.  Shows that the pins constrain every step of the oracle
(rotation, summaries, codes, lists, eligibility, rerank, attention) and the
near-tie machinery that decides which GPU disagreements are excused
(margins, scales, threshold)."""
import itertools

import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import oracle_pins as pins


def _rope_wrong_sign(x, base):
    B, S, H, D = x.shape
    th = O.rope_angles(S, D, base).astype(np.float64)
    c, s = np.cos(th)[None, :, None, :], np.sin(th)[None, :, None, :]
    x1, x2 = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([x1 * c + x2 * s, x2 * c - x1 * s], axis=-1)


def _rope_interleaved(x, base):
    B, S, H, D = x.shape
    th = O.rope_angles(S, D, base).astype(np.float64)
    c, s = np.cos(th)[None, :, None, :], np.sin(th)[None, :, None, :]
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _means_as_sums(xr, bs):
    B, S, H, D = xr.shape
    return xr.reshape(B, S // bs, bs, H, D).sum(axis=2).transpose(0, 2, 1, 3)


def _codes_argmin(kbar, codebooks):
    P, K, _ = codebooks.shape
    sc = O.codeword_scores(kbar, codebooks)
    codes = np.argmin(sc, axis=-1)
    addr = (codes * K ** np.arange(P - 1, -1, -1)).sum(axis=-1)
    return addr, codes, np.zeros(sc.shape[:-1])


def _codes_last_subspace_major(kbar, codebooks):
    P, K, _ = codebooks.shape
    sc = O.codeword_scores(kbar, codebooks)
    codes = np.argmax(sc, axis=-1)
    addr = (codes * K ** np.arange(P)).sum(axis=-1)
    return addr, codes, np.zeros(sc.shape[:-1])


def _lists_keep_latest(addr_row, A, cap):
    lists = np.full((A, cap), -1, dtype=np.int64)
    load = np.zeros(A, dtype=np.int64)
    for i, a in enumerate(addr_row):
        if load[a] >= cap:
            lists[a, :-1] = lists[a, 1:]
            lists[a, -1] = i
        else:
            lists[a, load[a]] = i
        load[a] += 1
    return lists, load, int(np.maximum(load - cap, 0).sum()), int(load.max())


def _slots_off_by_one(lists, probe_addrs, j, L):
    slots = lists[probe_addrs].copy()
    slots[(slots < 0) | (slots > j - L + 1)] = -1
    return slots


def _route_row_lowest_scores(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    slots = O.candidate_slots(lists, probe_addrs, j, L)
    cand = slots[slots >= 0]
    scores = O.f32(O.f32(kbar_h[cand]) @ O.f32(qbar_j)) if cand.size else np.zeros(0)
    order = np.lexsort((cand, scores))                    # ascending: wrong end
    top = cand[order[:R]]
    remote = np.full(R, -1, dtype=np.int64)
    remote[: top.size] = np.sort(top)
    local = np.arange(j - L + 1, j + 1)
    local[local < 0] = -1
    return O.RouteRow(np.concatenate([remote, local]), slots, cand, scores, np.inf,
                      float(np.abs(scores).max()) if scores.size else 0.0)


def _make_attend(scale_mult=1.0, causal=True, kv_map=lambda hq, g, Hkv: hq // g):
    def attend(qr, kr, v, sel, bs, scale, rows=None):
        B, S, Hq, D = qr.shape
        Hkv = kr.shape[2]
        g = Hq // Hkv
        out = np.full((B, S, Hq, v.shape[3]), np.nan)
        for b, hq, j in itertools.product(range(B), range(Hq), range(S // bs)):
            toks = O.selected_tokens(sel[b, hq, j], bs)
            qpos = np.arange(j * bs, (j + 1) * bs)
            h = kv_map(hq, g, Hkv)
            s = (qr[b, qpos, hq] @ kr[b, toks, h].T) * scale * scale_mult
            if causal:
                s[toks[None, :] > qpos[:, None]] = -np.inf
            s -= s.max(axis=1, keepdims=True)
            w = np.exp(s)
            out[b, qpos, hq] = (w @ v[b, toks, h]) / w.sum(axis=1, keepdims=True)
        return out
    return attend


# ---- mistakes in the near-tie machinery (margins, scales, threshold): each
# would excuse real disagreements between the GPU and the oracle
_REAL_ASSIGN = O.assign_codes
_REAL_PROBE = O.probe_codes
_REAL_ROUTE_ROW = O.route_row
_REAL_NEAR_TIE = O.near_tie
_REAL_CODE_SCALE = O.code_scale


def _code_margin_zero(kbar, codebooks):
    addr, codes, margin = _REAL_ASSIGN(kbar, codebooks)
    return addr, codes, np.zeros_like(margin)


def _code_margin_wrong_ranks(kbar, codebooks):
    addr, codes, _ = _REAL_ASSIGN(kbar, codebooks)
    srt = -np.sort(-O.codeword_scores(kbar, codebooks), axis=-1)
    return addr, codes, (srt[..., 1] - srt[..., 2]) if srt.shape[-1] > 2 else np.full(srt.shape[:-1], np.inf)


def _probe_margin_wrong_ranks(qbar, codebooks, p):
    codes, _ = _REAL_PROBE(qbar, codebooks, p)
    srt = -np.sort(-O.codeword_scores(qbar, codebooks), axis=-1)
    return codes, srt[..., 0] - srt[..., 1]


def _route_margin_wrong_ranks(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    row = _REAL_ROUTE_ROW(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force)
    srt = np.sort(row.scores)[::-1]
    row.margin = float(srt[R] - srt[R + 1]) if srt.size > R + 1 else np.inf   # one rank too deep
    return row


def _route_margin_zero(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    row = _REAL_ROUTE_ROW(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force)
    row.margin = 0.0
    return row


def _route_scale_zero(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    row = _REAL_ROUTE_ROW(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force)
    row.scale = 0.0
    return row


def _code_scale_signed(xbar, codebooks):
    return O.codeword_scores(xbar, codebooks).max(axis=-1)       # largest score, not |score|


MUTATIONS = {
    "code_margin_always_zero": ("assign_codes", _code_margin_zero),
    "code_margin_wrong_ranks": ("assign_codes", _code_margin_wrong_ranks),
    "probe_margin_wrong_ranks": ("probe_codes", _probe_margin_wrong_ranks),
    "route_margin_wrong_ranks": ("route_row", _route_margin_wrong_ranks),
    "route_margin_always_zero": ("route_row", _route_margin_zero),
    "route_scale_zero": ("route_row", _route_scale_zero),
    "code_scale_signed": ("code_scale", _code_scale_signed),
    "near_tie_threshold_loose": ("near_tie", lambda m, s: np.asarray(m) < 1e-3 * np.maximum(1.0, np.abs(s))),
    "near_tie_threshold_absolute": ("near_tie", lambda m, s: np.asarray(m) < 1e-6 + 0 * np.asarray(s)),

    "rope_rotates_backwards": ("rope", _rope_wrong_sign),
    "rope_interleaved_pairs": ("rope", _rope_interleaved),
    "summary_is_sum": ("block_means", _means_as_sums),
    "codes_argmin": ("assign_codes", _codes_argmin),
    "address_last_subspace_major": ("assign_codes", _codes_last_subspace_major),
    "lists_keep_latest": ("build_lists", _lists_keep_latest),
    "eligibility_off_by_one": ("candidate_slots", _slots_off_by_one),
    "rerank_lowest_scores": ("route_row", _route_row_lowest_scores),
    "attention_no_scale": ("attend", _make_attend(scale_mult=np.sqrt(16.0))),
    "attention_not_causal": ("attend", _make_attend(causal=False)),
    "attention_wrong_kv_head": ("attend", _make_attend(kv_map=lambda hq, g, Hkv: hq % Hkv)),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check()
        except AssertionError:
            caught.append(check.__name__)
    assert caught, f"no pin catches the mutation {name}"
