"""GPU parity of the controls and diagnostics: mdr_route_forced (the
forced-target route; "Monodratic Claims Learned Routing Can Make Sparse
Causal Attention More Selective", section "Why Learned Product-Hash Routing
Matters Now") and mdr_target_hits (the target-block hit rate; "Monodratic: a
reproducible sparse attention mixer", section Evidence), against the
oracle's route(force=...) and target_hits on the same seeded inputs, with
the bar of tests/parity_util.py (selected ids and hit counts bit-exact
outside near ties)."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from tests import parity_util as U
from workloads import AR, CAPACITY, SCALING_32K, TINY, make_inputs

pytestmark = pytest.mark.gpu


def mixed_targets(w, seed):
    """A forced id per route: half of them a remote-eligible block (where
    one exists), the rest -1, the own block, a later block or an id past the
    end."""
    rng = np.random.default_rng(seed)
    shape = (w.B, w.Hq, w.nb)
    j = np.broadcast_to(np.arange(w.nb), shape)
    kind = rng.integers(0, 8, size=shape)
    elig = np.floor(rng.random(shape) * np.maximum(j - w.L + 1, 1)).astype(np.int64)
    t = np.full(shape, -1, dtype=np.int64)
    t = np.where((kind <= 3) & (j - w.L >= 0), elig, t)
    t = np.where(kind == 4, j, t)
    t = np.where(kind == 5, np.minimum(j + 1, w.nb - 1), t)
    t = np.where(kind == 6, w.nb + 7, t)
    return t


def planted_targets(w, inp):
    """The planted block of each sequence as the target of the last query
    block of every head (the workload's retrieval question); -1 elsewhere."""
    t = np.full((w.B, w.Hq, w.nb), -1, dtype=np.int64)
    t[:, :, w.nb - 1] = inp.planted[:, None]
    return t


def gpu_hits(w, sel, target):
    import torch
    from learned_product_hash_b200 import mdr
    cfg = mdr.make_config(w)
    s = torch.from_numpy(np.ascontiguousarray(sel, dtype=np.int32)).cuda()
    t = torch.from_numpy(np.ascontiguousarray(target, dtype=np.int32)).cuda()
    hit = torch.full(target.shape, 99, dtype=torch.int32, device="cuda")
    counts = torch.full((2,), -7, dtype=torch.int32, device="cuda")
    mdr.mdr_target_hits(cfg, s, t, counts, hit)
    return hit.cpu().numpy(), [int(x) for x in counts.cpu()]


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("w", [TINY, AR.with_(B=8), CAPACITY], ids=lambda w: w.name)
def test_forced_route_matches_oracle(w, seed):
    """Forced ids of every kind (eligible, none, local, later, past the end):
    index, probes, selected blocks, candidate counts and attention as the
    oracle's forced route; every eligible target is selected."""
    inp = make_inputs(w, seed)
    tg = mixed_targets(w, 10 + seed)
    g = U.run_gpu(w, inp, "forced", tg)
    res = U.oracle_for(w, inp, force=tg)
    rep = U.compare(w, g, res, inp.codebooks, force=tg, max_ties=2)
    print(f"ties forced {w.name} seed {seed}: {rep}")
    j = np.arange(w.nb)[None, None, :]
    elig = (tg >= 0) & (tg <= j - w.L) & (w.R > 0)
    got = (g["sel"][..., : w.R] == tg[..., None]).any(axis=-1)
    assert got[elig].all()


@pytest.mark.parametrize("w", [TINY, AR, CAPACITY], ids=lambda w: w.name)
def test_target_hits_bit_exact(w):
    """Hits of the GPU's own routes against the oracle's count on the same
    rows: per route and in total (the planted-block workload has 1536
    routes, more than the kernel's 1024 threads); no target at all gives
    (0, 0)."""
    inp = make_inputs(w, 4)
    g = U.run_gpu(w, inp)
    tg = mixed_targets(w, 5)
    hit, counts = gpu_hits(w, g["sel"], tg)
    ref_hit, n, nh = O.target_hits(g["sel"], tg)
    assert np.array_equal(hit, ref_hit)
    assert counts == [n, nh]
    none = np.full_like(tg, -1)
    hit, counts = gpu_hits(w, g["sel"], none)
    assert counts == [0, 0] and (hit == -1).all()


def test_planted_block_controls():
    """The planted-block workload's three routes, as in the pages' controls:
    the route with random codebooks (the untrained router) finds the planted
    block as often as the oracle's route does; forcing it gives every hit;
    the local-only control (R = 0) never finds it."""
    w = AR
    inp = make_inputs(w, 0)
    tg = planted_targets(w, inp)
    g = U.run_gpu(w, inp)
    res = U.oracle_for(w, inp, rows=[])
    _, counts = gpu_hits(w, g["sel"], tg)
    _, n, nh = O.target_hits(res.sel, tg)
    last_tie = O.near_tie(res.sel_margin[:, :, -1], res.sel_scale[:, :, -1]).sum() + \
        O.near_tie(res.qcode_margin[:, :, -1], np.abs(O.codeword_scores(res.qbar[:, :, -1], inp.codebooks)).max(-1)).any(-1).sum()
    assert counts[0] == n == w.B * w.Hq
    assert abs(counts[1] - nh) <= last_tie
    assert 0 < counts[1] < n                      # random codebooks find it sometimes, not always
    gf = U.run_gpu(w, inp, "forced", tg)
    _, counts_f = gpu_hits(w, gf["sel"], tg)
    assert counts_f == [n, n]
    wl = w.with_(R=0)
    gl = U.run_gpu(wl, inp)
    _, counts_l = gpu_hits(wl, gl["sel"], tg)
    assert counts_l == [n, 0]


def test_forced_route_full_size_sampled():
    """The 32K workload with mixed forced ids: routing compared everywhere,
    attention on sampled query blocks."""
    w = SCALING_32K
    inp = make_inputs(w, 0)
    tg = mixed_targets(w, 6)
    g = U.run_gpu(w, inp, "forced", tg)
    p = O.Params.of(w)
    res = O.forward(inp.q, inp.k, inp.v, inp.codebooks, p, attention=False, force=tg)
    rows = U.sampled_rows(w, res)
    res.out = O.attend(res.qr, res.kr, res.v, res.sel, w.block, p.softmax_scale, rows)
    rep = U.compare(w, g, res, inp.codebooks, force=tg, max_ties=U.full_size_tie_budget(w))
    print(f"ties forced {w.name}: {rep}")
