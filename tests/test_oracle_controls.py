"""The oracle's controls and diagnostics (no GPU): the forced-target route
(Article, "Why Learned Product-Hash Routing Matters Now": the labelled target
block put into the selected set under the same attention budget), the
local-only control (R = 0; Report, Learned sparse route) and the
target-block hit count (Report, Evidence)."""
import numpy as np
import pytest

from oracle import mdr_oracle as O


def _p(**kw):
    base = dict(B=1, S=128, Hq=2, Hkv=1, D=32, block=16, P=2, K=4, cap=8,
                probes=2, R=3, L=1, rope_base=10000.0, scale=0.0)
    base.update(kw)
    return O.Params(**base)


def _inputs(p, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((p.B, p.S, p.Hq, p.D))
    k = rng.standard_normal((p.B, p.S, p.Hkv, p.D))
    v = rng.standard_normal((p.B, p.S, p.Hkv, p.D))
    c = rng.standard_normal((p.P, p.K, p.D // p.P))
    c = (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)
    return q, k, v, c


def _targets(p, seed):
    """A forced id per route: a random eligible block where one exists, and
    some routes with -1, a local block or a later block."""
    rng = np.random.default_rng(seed)
    t = np.full((p.B, p.Hq, p.nb), -1, dtype=np.int64)
    for b in range(p.B):
        for h in range(p.Hq):
            for j in range(p.nb):
                kind = rng.integers(0, 6)
                if kind <= 2 and j - p.L >= 0:
                    t[b, h, j] = rng.integers(0, j - p.L + 1)
                elif kind == 3:
                    t[b, h, j] = j                       # a local block
                elif kind == 4:
                    t[b, h, j] = min(j + 1, p.nb - 1)    # a later block (or the own one)
    return t


def test_forced_route_equals_brute_force_when_every_block_is_a_candidate():
    """With every address probed (p = K) and lists holding every block
    (cap >= nb), the forced route is: the target plus the R - 1 best other
    eligible blocks by <qbar_j, kbar_i>, found here by sorting the full score
    matrix with Python's sorted()."""
    p = _p(K=2, probes=2, cap=16, R=3, L=1)
    q, k, v, c = _inputs(p, 1)
    tg = _targets(p, 2)
    r = O.forward(q, k, v, c, p, attention=False, force=tg)
    for h in range(p.Hq):
        for j in range(p.nb):
            f = int(tg[0, h, j])
            elig = list(range(0, j - p.L + 1))
            sc = {i: float(np.float32(np.dot(np.float32(r.qbar[0, h, j]), np.float32(r.kbar[0, 0, i]))))
                  for i in elig}
            if 0 <= f <= j - p.L:
                rest = sorted((i for i in elig if i != f), key=lambda i: (-sc[i], i))[: p.R - 1]
                want = sorted(rest + [f])
            else:
                want = sorted(sorted(elig, key=lambda i: (-sc[i], i))[: p.R])
            want = want + [-1] * (p.R - len(want))
            assert list(r.sel[0, h, j, : p.R]) == want, (h, j, f)


def test_forced_target_replaces_the_weakest_choice_or_changes_nothing():
    """Against the unforced route: a target it already selected leaves the
    row unchanged; a target it missed takes the place of its lowest-scored
    remote choice (or of a -1 pad); a target that is not remote-eligible
    changes nothing.  Small lists (cap 1) make misses common."""
    p = _p(K=4, probes=2, cap=1, R=2, L=1, S=256)
    q, k, v, c = _inputs(p, 3)
    tg = _targets(p, 4)
    base = O.forward(q, k, v, c, p, attention=False)
    forc = O.forward(q, k, v, c, p, attention=False, force=tg)
    n_missed = 0
    for h in range(p.Hq):
        for j in range(p.nb):
            f = int(tg[0, h, j])
            b_rem = [x for x in base.sel[0, h, j, : p.R] if x >= 0]
            f_rem = [x for x in forc.sel[0, h, j, : p.R] if x >= 0]
            assert list(forc.sel[0, h, j, p.R:]) == list(base.sel[0, h, j, p.R:])
            if not (0 <= f <= j - p.L) or f in b_rem:
                assert list(forc.sel[0, h, j]) == list(base.sel[0, h, j]), (h, j)
                continue
            n_missed += 1
            sc = {i: float(np.float32(np.dot(np.float32(base.qbar[0, h, j]), np.float32(base.kbar[0, 0, i]))))
                  for i in b_rem}
            if len(b_rem) == p.R:
                weakest = sorted(b_rem, key=lambda i: (-sc[i], i))[-1]
                want = sorted([x for x in b_rem if x != weakest] + [f])
            else:
                want = sorted(b_rem + [f])
            assert f_rem == want, (h, j, f, b_rem, f_rem)
    assert n_missed > 5


def test_forcing_with_no_remote_budget_changes_nothing():
    """Local-only control (R = 0): there is no remote slot to force into."""
    p = _p(R=0, L=2)
    q, k, v, c = _inputs(p, 5)
    tg = _targets(p, 6)
    a = O.forward(q, k, v, c, p, attention=False)
    b = O.forward(q, k, v, c, p, attention=False, force=tg)
    assert np.array_equal(a.sel, b.sel)


def test_target_hits_on_a_hand_counted_fixture():
    """Selected rows and targets written out by hand, hits counted by hand."""
    sel = np.array([[[[0, 3, 5], [-1, -1, 1], [2, 4, 5], [1, 2, 3]],
                     [[0, 1, 4], [1, -1, 3], [-1, -1, 0], [4, -1, 6]]]])
    target = np.array([[[3, 0, -1, 3],
                        [2, 3, -1, -1]]])
    hit, n, nh = O.target_hits(sel, target)
    assert hit.tolist() == [[[1, 0, -1, 1], [0, 1, -1, -1]]]
    assert (n, nh) == (5, 3)


def test_forced_route_always_hits_and_local_only_never_hits_a_remote_target():
    """Forcing the target makes every route with an eligible target hit it
    (the Article's forced diagnostic recovers every miss); the local-only
    control (R = 0) never selects a remote target."""
    p = _p(K=4, probes=1, cap=2, R=2, L=1, S=256)
    q, k, v, c = _inputs(p, 7)
    rng = np.random.default_rng(8)
    tg = np.full((p.B, p.Hq, p.nb), -1, dtype=np.int64)
    for j in range(p.L, p.nb):
        tg[0, :, j] = rng.integers(0, j - p.L + 1, size=p.Hq)
    free = O.forward(q, k, v, c, p, attention=False)
    forc = O.forward(q, k, v, c, p, attention=False, force=tg)
    loc = O.forward(q, k, v, c, p.__class__(**{**p.__dict__, "R": 0}), attention=False)
    _, n, nh_free = O.target_hits(free.sel, tg)
    _, n2, nh_forc = O.target_hits(forc.sel, tg)
    _, n3, nh_loc = O.target_hits(loc.sel, tg)
    assert n == n2 == n3 == p.Hq * (p.nb - p.L)
    assert nh_forc == n
    assert nh_loc == 0
    assert nh_free < n                  # one probe, two slots: routing misses some


@pytest.mark.parametrize("R", [1, 2, 4])
def test_forced_route_is_causal(R):
    """Forcing never brings in a block later than j - L: ids outside the
    eligible range are ignored."""
    p = _p(R=R)
    q, k, v, c = _inputs(p, 9)
    tg = _targets(p, 10)
    r = O.forward(q, k, v, c, p, attention=False, force=tg)
    for j in range(p.nb):
        rem = r.sel[0, :, j, : p.R]
        assert (rem[rem >= 0] <= j - p.L).all()


# ------------------------------------------------ planted mistakes are caught
def _forced_replaces_the_best(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    row = _ROUTE_ROW(qbar_j, kbar_h, probe_addrs, lists, j, R, L)
    if not (0 <= force <= j - L and R > 0):
        return row
    rem = [x for x in row.sel[:R] if x >= 0]
    if force in rem:
        return row
    if len(rem) == R:                              # drop the best instead of the weakest
        sc = {i: float(np.float32(np.dot(np.float32(qbar_j), np.float32(kbar_h[i])))) for i in rem}
        rem.remove(sorted(rem, key=lambda i: (-sc[i], i))[0])
    rem = sorted(rem + [force])
    row.sel[:R] = rem + [-1] * (R - len(rem))
    return row


def _forced_ignores_eligibility(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force=-1):
    row = _ROUTE_ROW(qbar_j, kbar_h, probe_addrs, lists, j, R, L, force)
    if R > 0 and force > j - L:                    # a local or later block forced in anyway
        rem = sorted([x for x in row.sel[:R] if x >= 0][: R - 1] + [force])
        row.sel[:R] = rem + [-1] * (R - len(rem))
    return row


def _hits_count_untargeted_routes(sel, target):
    hit, n, nh = _TARGET_HITS(sel, target)
    return hit, target.size, nh


_ROUTE_ROW = O.route_row
_TARGET_HITS = O.target_hits
CONTROL_CHECKS = [
    test_forced_route_equals_brute_force_when_every_block_is_a_candidate,
    test_forced_target_replaces_the_weakest_choice_or_changes_nothing,
    test_forcing_with_no_remote_budget_changes_nothing,
    test_target_hits_on_a_hand_counted_fixture,
    test_forced_route_always_hits_and_local_only_never_hits_a_remote_target,
    lambda: [test_forced_route_is_causal(R) for R in (1, 2, 4)],
]


@pytest.mark.parametrize("attr,fn", [("route_row", _forced_replaces_the_best),
                                     ("route_row", _forced_ignores_eligibility),
                                     ("target_hits", _hits_count_untargeted_routes)])
def test_control_mutation_is_caught(attr, fn, monkeypatch):
    monkeypatch.setattr(O, attr, fn)
    caught = 0
    for check in CONTROL_CHECKS:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no check catches {fn.__name__}"
