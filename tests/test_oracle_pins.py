"""The CPU oracle against closed forms, stated invariants, brute force and
library routines (no GPU)."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import oracle_pins as pins
from workloads import AR, CAPACITY, make_inputs


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(check):
    check()


def test_planted_block_is_found():
    """Sanity of the associative-recall-shaped workload: the planted block is
    the best-scoring eligible block for the last query block almost always,
    and the untrained (random-codebook) router still selects it often."""
    w = AR.with_(B=16)
    inp = make_inputs(w, 0)
    p = O.Params.of(w)
    res = O.forward(inp.q, inp.k, inp.v, inp.codebooks, p, attention=False)
    nb = w.nb
    hits_route, hits_best = [], []
    for b in range(w.B):
        for h in range(w.Hq):
            sc = res.qbar[b, h, nb - 1] @ res.kbar[b, h // (w.Hq // w.Hkv), : nb - w.L].T
            hits_best.append(int(np.argmax(sc)) == inp.planted[b])
            hits_route.append(inp.planted[b] in res.sel[b, h, nb - 1, : w.R])
    assert np.mean(hits_best) > 0.95
    assert np.mean(hits_route) > 0.3


def test_planted_block_mean_cosine_is_the_stated_one():
    """The planted-block workload states that the planted block's mean key
    aligns with cosine 0.9 with the last block's mean query: measured here on
    the rotated block means (the oracle's), averaged over sequences and
    heads."""
    w = AR.with_(B=32)
    inp = make_inputs(w, 0)
    res = O.forward(inp.q, inp.k, inp.v, inp.codebooks, O.Params.of(w), attention=False)
    cs = []
    for b in range(w.B):
        for h in range(w.Hq):
            qb, kb = res.qbar[b, h, w.nb - 1], res.kbar[b, h, inp.planted[b]]
            cs.append(qb @ kb / np.linalg.norm(qb) / np.linalg.norm(kb))
    assert abs(np.mean(cs) - 0.9) < 0.01, np.mean(cs)


def test_capacity_workload_load():
    """The capacity workload has the report's capacity-run shape (8,192
    tokens, capacity 64); its lists stay under capacity."""
    inp = make_inputs(CAPACITY, 0)
    p = O.Params.of(CAPACITY)
    kr = O.rope(inp.k.astype(np.float64), p.rope_base)
    _, _, _, _, lists, load, ovf, mx = O.build_index(kr, inp.codebooks, p)
    assert (ovf == 0).all() and (mx <= CAPACITY.cap).all()
    assert (load.sum(axis=-1) == CAPACITY.nb).all()
