"""Pins of the equal-size spherical k-means oracle (FlashHead pages, Module 1, Eq.4 and Eq.5) to
facts that do not come from the oracle itself: brute-force enumeration of every equal-size
partition, the Cauchy-Schwarz closed form of the centre update, weak duality of the
transportation problem, invariances of cosine clustering, and recovery of planted clusters."""

import numpy as np
import pytest

from oracle import kmeans_oracle as K


def unit(a):
    return a / np.linalg.norm(a, axis=1, keepdims=True)


def planted(c, b, d, spread, seed):
    """c well-separated directions with exactly b noisy members each, token ids shuffled."""
    rng = np.random.default_rng(seed)
    centres = unit(rng.standard_normal((c, d)))
    lab = np.repeat(np.arange(c), b)
    X = centres[lab] + spread * rng.standard_normal((c * b, d)) / np.sqrt(d)
    X *= rng.uniform(0.5, 2.0, size=(c * b, 1))  # norms play no part in spherical clustering
    perm = rng.permutation(c * b)
    return X[perm].astype(np.float32), lab[perm]


def test_bf16_storage_is_read_exactly():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000], dtype=np.uint16)
    assert K.stored_to_f64(bits).tolist() == [1.0, -2.0, 1.0078125, 0.0, -0.0]


@pytest.mark.parametrize("v,c", [(6, 2), (6, 3), (6, 6), (8, 2), (8, 4)])
def test_assignment_is_the_best_equal_size_partition(v, c):
    """Linear assignment over replicated slots reaches the maximum found by enumerating every
    equal-size partition (b = 1 is the plain permutation case)."""
    rng = np.random.default_rng(v * 10 + c)
    for trial in range(3):
        X = unit(rng.standard_normal((v, 5)))
        C = unit(rng.standard_normal((c, 5)))
        lab = K.assign_equal_size(X, C, v // c)
        assert K.is_equal_size(lab, c, v // c)
        A = X @ C.T
        assert K.assignment_value(A, lab) == pytest.approx(K.brute_force_assignment(A, v // c),
                                                           abs=1e-12)


def test_assignment_is_nearest_centre_when_that_is_balanced():
    X, lab = planted(c=6, b=5, d=16, spread=0.05, seed=3)
    Xu = K.unit_rows(X)
    C = K.update_centres(Xu, lab, 6)
    nearest = np.argmax(Xu @ C.T, axis=1)
    assert np.array_equal(nearest, lab)
    assert np.array_equal(K.assign_equal_size(Xu, C, 5), lab)


def test_assignment_respects_capacity_against_nearest_centre():
    """All tokens nearest to one centre: the constraint must spill them to the others."""
    rng = np.random.default_rng(8)
    X = unit(np.array([1.0, 0.0, 0.0]) + 0.01 * rng.standard_normal((12, 3)))
    C = unit(np.array([[1.0, 0.0, 0.0], [0.0, 1.0, 0.0], [0.0, 0.0, 1.0]]))
    lab = K.assign_equal_size(X, C, 4)
    assert np.bincount(lab, minlength=3).tolist() == [4, 4, 4]
    # which four stay with centre 0 is fixed by optimality, checked by enumeration on six tokens
    small = X[:6]
    lab6 = K.assign_equal_size(small, C, 2)
    A = small @ C.T
    assert K.assignment_value(A, lab6) == pytest.approx(K.brute_force_assignment(A, 2), abs=1e-12)


def test_centre_update_reaches_the_cauchy_schwarz_bound():
    """Eq.5 maximises sum_{i in k} x_i . c over unit c; the maximum is |sum_{i in k} x_i|."""
    rng = np.random.default_rng(11)
    X = unit(rng.standard_normal((40, 7)))
    lab = rng.integers(0, 4, size=40)
    lab[:4] = np.arange(4)
    C = K.update_centres(X, lab, 4)
    for k in range(4):
        s = X[lab == k].sum(axis=0)
        assert float((X[lab == k] @ C[k]).sum()) == pytest.approx(float(np.linalg.norm(s)), rel=1e-13)
        for _ in range(20):
            other = unit((C[k] + 0.1 * rng.standard_normal(7))[None])[0]
            assert (X[lab == k] @ other).sum() <= (X[lab == k] @ C[k]).sum() + 1e-12
    assert np.allclose(np.linalg.norm(C, axis=1), 1.0, atol=1e-14)


def test_single_cluster_and_singletons():
    rng = np.random.default_rng(2)
    X = unit(rng.standard_normal((9, 4)))
    C1 = K.update_centres(X, np.zeros(9, dtype=np.int64), 1)
    m = X.mean(axis=0)
    assert np.allclose(C1[0], m / np.linalg.norm(m), atol=1e-15)
    Cs = K.update_centres(X, np.arange(9), 9)
    assert np.allclose(Cs, X, atol=1e-15)


def test_objective_never_rises():
    rng = np.random.default_rng(5)
    E = rng.standard_normal((96, 12)).astype(np.float32)
    lab, C, hist = K.kmeans(E, 8, init_tokens=rng.permutation(96)[:8], iters=50)
    assert K.is_equal_size(lab, 8, 12)
    assert all(b <= a + 1e-9 for a, b in zip(hist, hist[1:]))
    X = K.unit_rows(E)
    # the result is a fixed point: re-assigning with its own centres changes nothing of value
    A = X @ C.T
    assert K.assignment_value(A, K.assign_equal_size(X, C, 12)) == pytest.approx(
        K.assignment_value(A, lab), abs=1e-9)


def test_planted_clusters_are_recovered():
    X, lab = planted(c=8, b=16, d=32, spread=0.3, seed=7)
    init = np.array([np.nonzero(lab == k)[0][0] for k in range(8)])
    got, C, hist = K.kmeans(X, 8, init_tokens=init, iters=20)
    assert np.array_equal(got, lab)  # init token of cluster k is in cluster k, so labels match
    Xu = K.unit_rows(X)
    closed = -sum(np.linalg.norm(Xu[lab == k].sum(axis=0)) for k in range(8))
    assert hist[-1] == pytest.approx(closed, rel=1e-12)


def test_rotation_and_row_scaling_change_nothing():
    rng = np.random.default_rng(9)
    E = rng.standard_normal((48, 6))
    init = rng.permutation(48)[:6]
    lab, C, hist = K.kmeans(E, 6, init, iters=30)
    Q, _ = np.linalg.qr(rng.standard_normal((6, 6)))
    E2 = (E @ Q) * rng.uniform(0.1, 10.0, size=(48, 1))
    lab2, C2, hist2 = K.kmeans(E2, 6, init, iters=30)
    assert np.array_equal(lab, lab2)
    assert hist2[-1] == pytest.approx(hist[-1], rel=1e-10)
    assert np.allclose(C @ Q, C2, atol=1e-10)


def test_token_order_is_irrelevant():
    rng = np.random.default_rng(4)
    E = rng.standard_normal((40, 5))
    init = np.arange(0, 40, 8)
    lab, _, hist = K.kmeans(E, 5, init, iters=30)
    perm = rng.permutation(40)
    inv = np.argsort(perm)
    lab2, _, hist2 = K.kmeans(E[perm], 5, inv[init], iters=30)
    assert np.array_equal(lab2, lab[perm])
    assert hist2[-1] == pytest.approx(hist[-1], rel=1e-12)


def test_weak_duality_and_the_eps_certificate():
    """Any prices bound every equal-size assignment from above; a labeling whose slackness gap is
    g is within v * g of that bound, hence of the optimum."""
    rng = np.random.default_rng(12)
    v, c = 8, 4
    A = unit(rng.standard_normal((v, 3))) @ unit(rng.standard_normal((c, 3))).T
    best = K.brute_force_assignment(A, v // c)
    for _ in range(50):
        p = rng.normal(0, 0.5, size=c)
        assert K.dual_bound(A, p, v // c) >= best - 1e-12
        lab = rng.permutation(np.repeat(np.arange(c), v // c))
        g = K.eps_cs_gap(A, lab, p)
        assert K.assignment_value(A, lab) >= K.dual_bound(A, p, v // c) - v * g - 1e-12


def test_c2t_is_a_dense_permutation():
    rng = np.random.default_rng(6)
    lab = rng.permutation(np.repeat(np.arange(5), 7))
    T = K.c2t_from_labels(lab, 5, 7)
    assert T.shape == (5, 7)
    assert np.array_equal(np.sort(T.ravel()), np.arange(35))
    for k in range(5):
        assert np.all(lab[T[k]] == k) and np.all(np.diff(T[k]) > 0)
    with pytest.raises(ValueError):
        K.c2t_from_labels(np.zeros(35, dtype=np.int64), 5, 7)
