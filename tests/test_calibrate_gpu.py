"""GPU parity of mdr_calibrate_codebooks (spherical codebook calibration;
"Monodratic: a reproducible sparse attention mixer", section Capacity and
Figure 3) against the oracle's calibration_step on the same seeded records.

Bar: assignments and member counts bit-exact outside near ties (a record
whose float32 margin between its two best codewords is below
1e-6*max(1,|score|) may go either way; the codewords whose member set it
changes are then checked for unit norm only).  Codewords within 2e-5 per
component: the GPU sums unit vectors in float32, sequentially per warp
(at most a few hundred members) and then over chunks, so each component of
a normalised sum carries at most about (members per warp + chunks) * 2^-24
~ 1e-5 relative error.  Multi-round runs are compared round by round, each
GPU round against the oracle round started from the GPU's previous
codebooks, so a flipped near tie cannot compound."""
import numpy as np
import pytest

from oracle import mdr_oracle as O
from workloads import LONG, make_keys, make_records

pytestmark = pytest.mark.gpu
TOL_CB = 2e-5


def _unit_codebooks(P, K, dsub, seed):
    r = np.random.default_rng(seed)
    c = r.standard_normal((P, K, dsub))
    return (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)


def gpu_round(X, C, rounds=1, in_place=False):
    import torch
    from learned_product_hash_b200 import mdr
    N, D = X.shape
    P, K, _ = C.shape
    x = torch.from_numpy(np.ascontiguousarray(X)).cuda()
    cin = torch.from_numpy(np.ascontiguousarray(C)).cuda()
    cout = cin if in_place else torch.full_like(cin, np.nan)
    counts = torch.full((P, K), -1, dtype=torch.int32, device="cuda")
    assign = torch.full((N, P), -1, dtype=torch.int32, device="cuda")
    ws = mdr.calibrate_workspace(N, D, P, K)
    mdr.mdr_calibrate_codebooks(x, cin, cout, rounds, ws, counts=counts, assign=assign)
    torch.cuda.synchronize()
    return cout.cpu().numpy(), assign.cpu().numpy(), counts.cpu().numpy()


def compare_round(X, C, g_cb, g_assign, g_counts):
    """One GPU round from codebooks C against the oracle's round from C."""
    r = O.calibration_step(X, C)
    P, K, _ = C.shape
    best = np.abs(O.codeword_scores(X.astype(np.float64).reshape(1, 1, -1, X.shape[1]), C)[0, 0]).max(-1)
    tie = O.near_tie(r.margin, best)                           # [N,P]
    diff = g_assign != r.assign
    assert not (diff & ~tie).any(), f"{int((diff & ~tie).sum())} assignments differ outside near ties"
    nz = np.zeros_like(diff)
    dsub = X.shape[1] // P
    for s in range(P):
        nz[:, s] = np.abs(X[:, s * dsub:(s + 1) * dsub]).max(axis=1) > 0
    for s in range(P):
        touched = set(g_assign[diff[:, s] & nz[:, s], s]) | set(r.assign[diff[:, s] & nz[:, s], s])
        for k in range(K):
            if k in touched:
                assert abs(np.linalg.norm(g_cb[s, k]) - 1.0) < 1e-5
                continue
            assert g_counts[s, k] == r.counts[s, k], (s, k)
            np.testing.assert_allclose(g_cb[s, k], r.codebooks[s, k], rtol=0, atol=TOL_CB)
    return int((diff & tie).sum())


CASES = {
    # N, D, P, K, centres, sigma, zero rows, repeated rows
    "d64_p2_k16": (3000, 64, 2, 16, 10, 0.3, 5, 4),
    "dsub8_p4_k8": (1000, 32, 4, 8, 6, 0.4, 0, 0),
    "dsub128_p1_k128": (5000, 128, 1, 128, 40, 0.3, 3, 0),
    "ragged_d128_p2_k64": (777, 128, 2, 64, 20, 0.2, 1, 9),
    "tiny_n1": (1, 64, 2, 4, 1, 0.1, 0, 0),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_round_matches_oracle(name):
    N, D, P, K, nc, sg, zr, rr = CASES[name]
    X = make_records(N, D, nc, sg, 20, zero_rows=zr, repeat_rows=rr)
    C = _unit_codebooks(P, K, D // P, 21)
    g = gpu_round(X, C)
    ties = compare_round(X, C, *g)
    assert ties <= 2


def test_rounds_are_deterministic_and_each_matches_oracle():
    """Five rounds in one call equal five chained one-round calls bit for
    bit; every chained round matches the oracle round from the same
    codebooks; in place equals out of place."""
    X = make_records(4000, 64, 12, 0.35, 22, zero_rows=2)
    C0 = _unit_codebooks(2, 32, 32, 23)
    five, _, _ = gpu_round(X, C0, rounds=5)
    C = C0
    for _ in range(5):
        g = gpu_round(X, C)
        compare_round(X, C, *g)
        C = g[0]
    np.testing.assert_array_equal(five, C)
    inplace, _, _ = gpu_round(X, C0, rounds=5, in_place=True)
    np.testing.assert_array_equal(inplace, five)
    zero, _, _ = gpu_round(X, C0, rounds=0)
    np.testing.assert_array_equal(zero, C0)


def test_codeword_without_members_keeps_its_value():
    r = np.random.default_rng(24)
    X = np.abs(r.standard_normal((500, 64))).astype(np.float32)
    C = _unit_codebooks(2, 3, 32, 25)
    C[:, 0] = 1 / np.sqrt(32)
    C[:, 1] = -1 / np.sqrt(32)
    cb, _, counts = gpu_round(X, C)
    assert (counts[:, 1] == 0).all()
    np.testing.assert_array_equal(cb[:, 1], C[:, 1])


def test_long_workload_key_summaries_twenty_rounds():
    """The long workload's key summaries of one training sequence (1024
    blocks x 8 KV heads = 8192 records of 128) with 64 codewords per
    subspace: twenty rounds, each against the oracle; the calibrated
    codebooks lower the overflow of a held-out sequence's index (built by
    the oracle)."""
    w = LONG
    kv, _ = make_keys(w, 11)
    kr = O.rope(kv.astype(np.float64), w.rope_base)
    X = O.f32(O.block_means(kr, w.block)).astype(np.float32).reshape(-1, w.D)
    from workloads import make_codebooks
    C = make_codebooks(w, 12)
    C0 = C
    for _ in range(20):
        g = gpu_round(X, C)
        compare_round(X, C, *g)
        C = g[0]
    kh, _ = make_keys(w, 12)
    kbar_h = O.block_means(O.rope(kh.astype(np.float64), w.rope_base), w.block)
    p = O.Params.of(w)

    def overflow(cb):
        addr, _, _ = O.assign_codes(kbar_h, cb)
        return sum(O.build_lists(addr[0, h], p.A, p.cap)[2] for h in range(w.Hkv))
    assert overflow(C) < overflow(C0)
