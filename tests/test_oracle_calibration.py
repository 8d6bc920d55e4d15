"""The oracle's codebook calibration (spherical k-means per subspace;
"Monodratic: a reproducible sparse attention mixer", section Capacity and
Figure 3) pinned without a GPU: against scikit-learn's Lloyd step on unit
vectors, a fixed point, invariances and the monotone objective; planted
mistakes are caught."""
import warnings

import numpy as np
import pytest

from oracle import mdr_oracle as O
from workloads import make_records


def _unit_codebooks(P, K, dsub, seed):
    r = np.random.default_rng(seed)
    c = r.standard_normal((P, K, dsub))
    return (c / np.linalg.norm(c, axis=-1, keepdims=True)).astype(np.float32)


def check_one_round_is_a_lloyd_step_on_unit_vectors():
    """Spherical assignment (largest cosine) is Euclidean nearest-centroid on
    unit vectors (|u - c|^2 = 2 - 2<u,c>), and the spherical update is the
    Euclidean mean of the unit members, normalised.  So one round equals
    scikit-learn's KMeans with init = the codebook, one Lloyd iteration, on
    x_s/|x_s|, followed by normalising its centres."""
    from sklearn.cluster import KMeans
    P, K, D = 2, 4, 32
    X = make_records(600, D, 5, 0.3, 1)
    C = _unit_codebooks(P, K, D // P, 2)
    st = O.calibration_step(X, C)
    assert (st.counts > 0).all()
    assert (st.margin > 1e-4).all()            # no near tie, so float64 and float32 decisions agree
    for s in range(P):
        Xs = X[:, s * 16:(s + 1) * 16].astype(np.float64)
        U = Xs / np.linalg.norm(Xs, axis=1, keepdims=True)
        with warnings.catch_warnings():
            warnings.simplefilter("ignore")
            km = KMeans(n_clusters=K, init=C[s].astype(np.float64), n_init=1, max_iter=1,
                        algorithm="lloyd", tol=0.0).fit(U)
        ref = km.cluster_centers_ / np.linalg.norm(km.cluster_centers_, axis=1, keepdims=True)
        np.testing.assert_allclose(st.codebooks[s], ref, rtol=0, atol=1e-12)


def check_codewords_are_a_fixed_point_of_their_own_copies():
    """Records that are positive multiples of the codewords (each codeword
    in one subspace paired with an arbitrary one in the other) leave the
    codebook unchanged; counts are the multiplicities."""
    P, K, dsub = 2, 6, 8
    C = np.zeros((P, K, dsub), dtype=np.float32)
    for s in range(P):
        for k in range(K):            # signed basis: +e_0, -e_0, +e_1, -e_1, ...
            C[s, k, k // 2] = 1.0 if k % 2 == 0 else -1.0
    r = np.random.default_rng(3)
    mult = r.integers(1, 5, size=K)
    rows = []
    for k in range(K):
        for _ in range(mult[k]):
            rows.append(np.concatenate([C[0, k] * r.uniform(0.5, 3.0), C[1, (k + 2) % K] * r.uniform(0.5, 3.0)]))
    st = O.calibration_step(np.array(rows, dtype=np.float32), C)
    np.testing.assert_array_equal(st.codebooks, C)
    assert list(st.counts[0]) == list(mult)
    assert list(st.counts[1]) == [mult[(k - 2) % K] for k in range(K)]


def check_zero_rows_are_ignored_and_copies_count():
    """Zero records have no direction: adding them changes neither the
    codebooks nor the counts.  An exact copy of a record counts twice."""
    P, K, D = 2, 5, 64
    X = make_records(300, D, 4, 0.3, 4)
    C = _unit_codebooks(P, K, D // P, 5)
    a = O.calibration_step(X, C)
    Xz = np.concatenate([X, np.zeros((7, D), dtype=np.float32)])
    b = O.calibration_step(Xz, C)
    np.testing.assert_array_equal(a.codebooks, b.codebooks)
    np.testing.assert_array_equal(a.counts, b.counts)
    Xd = np.concatenate([X, X[:1]])
    d = O.calibration_step(Xd, C)
    for s in range(P):
        k = a.assign[0, s]
        assert d.counts[s, k] == a.counts[s, k] + 1


def check_a_codeword_without_members_keeps_its_value():
    """Records confined to the positive orthant never choose the codeword
    -(1,...,1)/sqrt(d) when +(1,...,1)/sqrt(d) is offered: it keeps its value."""
    P, dsub = 2, 8
    r = np.random.default_rng(6)
    X = np.abs(r.standard_normal((200, P * dsub))).astype(np.float32)
    C = _unit_codebooks(P, 3, dsub, 7)
    C[:, 0] = 1 / np.sqrt(dsub)
    C[:, 1] = -1 / np.sqrt(dsub)
    st = O.calibration_step(X, C)
    assert (st.counts[:, 1] == 0).all()
    np.testing.assert_array_equal(st.codebooks[:, 1], C[:, 1])


def check_objective_never_decreases():
    """Spherical k-means does not decrease the summed cosine to the best
    codeword (assignment maximises it for fixed codewords; the normalised
    sum maximises it for fixed members)."""
    X = make_records(2000, 64, 12, 0.4, 8)
    C = _unit_codebooks(2, 16, 32, 9)
    prev = O.spherical_objective(X, C)
    for _ in range(8):
        C = O.calibration_step(X, C).codebooks
        cur = O.spherical_objective(X, C)
        assert cur >= prev - 1e-9
        prev = cur


def check_unit_rows_and_assignment_is_code_assignment():
    """Calibrated rows are unit vectors; the assignment is the address code
    of section 3 (assign_codes) of each record."""
    X = make_records(500, 128, 6, 0.2, 10)
    C = _unit_codebooks(2, 32, 64, 11)
    st = O.calibration_step(X, C)
    np.testing.assert_allclose(np.linalg.norm(st.codebooks, axis=-1), 1.0, atol=1e-12)
    _, codes, _ = O.assign_codes(X.astype(np.float64).reshape(1, 1, 500, 128), C)
    np.testing.assert_array_equal(st.assign, codes[0, 0])


CHECKS = [check_one_round_is_a_lloyd_step_on_unit_vectors, check_codewords_are_a_fixed_point_of_their_own_copies,
          check_zero_rows_are_ignored_and_copies_count, check_a_codeword_without_members_keeps_its_value,
          check_objective_never_decreases, check_unit_rows_and_assignment_is_code_assignment]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_calibration_pin(check):
    check()


# ------------------------------------------------ planted mistakes are caught
_STEP = O.calibration_step


def _mutant(kind):
    def step(records, codebooks):
        X = np.asarray(records, dtype=np.float64)
        C = np.asarray(codebooks, dtype=np.float64)
        P, K, dsub = C.shape
        sc = O.codeword_scores(X.reshape(1, 1, -1, P * dsub), C)[0, 0]
        assign = (np.argmin if kind == "argmin" else np.argmax)(sc, axis=-1)
        new = C.copy()
        counts = np.zeros((P, K), dtype=np.int64)
        for s in range(P):
            Xs = X[:, s * dsub:(s + 1) * dsub]
            n = np.linalg.norm(Xs, axis=1)
            for k in range(K):
                m = (assign[:, s] == k) & ((n >= 0) if kind == "count_zero_rows" else (n > 0))
                counts[s, k] = m.sum()
                if m.sum() == 0:
                    if kind == "empty_zeroed":
                        new[s, k] = 0.0
                    continue
                u = Xs[m] if kind == "raw_sum" else Xs[m] / np.maximum(n[m, None], 1e-300)
                t = u.sum(axis=0)
                new[s, k] = t if kind == "no_normalise" else t / np.linalg.norm(t)
        return O.CalibStep(new, assign, np.full((X.shape[0], P), np.inf), counts)
    return step


@pytest.mark.parametrize("kind", ["argmin", "raw_sum", "no_normalise", "empty_zeroed", "count_zero_rows"])
def test_calibration_mutation_is_caught(kind, monkeypatch):
    monkeypatch.setattr(O, "calibration_step", _mutant(kind))
    caught = 0
    for check in CHECKS:
        try:
            check()
        except AssertionError:
            caught += 1
    assert caught, f"no calibration check catches {kind}"
