"""Pins of the k-means warm-start oracle (oracle/kmeans_oracle.py) to things other than
itself: an independent distance routine, scalar brute force on tiny inputs, closed
forms, the exact sampling law of the seeding draw and Lloyd's monotone inertia."""
import numpy as np
import pytest
from scipy.spatial.distance import cdist

from oracle import kmeans_oracle as KM


def test_fp32_distances_match_scipy_within_fp32_rounding():
    rng = np.random.default_rng(0)
    X = rng.normal(size=(200, 37)).astype(np.float32) * 3
    C = rng.normal(size=(11, 37)).astype(np.float32) * 3
    ref = cdist(X.astype(np.float64), C.astype(np.float64), "sqeuclidean")
    got = KM.sqdist_fp32(X, C).astype(np.float64)
    assert np.max(np.abs(got - ref) / np.maximum(ref, 1e-30)) < 37 * 2.0 ** -22


def test_fp32_distances_are_the_stated_operation_sequence():
    """Scalar restatement on a tiny input: per dimension in order, subtract, square and
    add, each rounded to fp32 (no fused multiply-add)."""
    rng = np.random.default_rng(1)
    X = (rng.normal(size=(5, 7)) * 10).astype(np.float32)
    C = (rng.normal(size=(3, 7)) * 10).astype(np.float32)
    got = KM.sqdist_fp32(X, C)
    for i in range(5):
        for k in range(3):
            acc = np.float32(0)
            for d in range(7):
                t = np.float32(X[i, d] - C[k, d])
                acc = np.float32(acc + np.float32(t * t))
            assert got[i, k] == acc


def test_assignment_brute_force_and_lowest_index_on_ties():
    X = np.array([[0, 0], [1, 0], [3, 0], [2, 0]], dtype=np.float32)
    C = np.array([[1, 0], [3, 0], [1, 0]], dtype=np.float32)   # centres 0 and 2 coincide
    a, d = KM.assign(X, C)
    # (2, 0) is equally far from centres 0/2 and 1: the lowest index wins
    np.testing.assert_array_equal(a, [0, 0, 1, 0])
    np.testing.assert_array_equal(d, [1, 0, 0, 1])


def test_lloyd_step_closed_form_two_blobs():
    rng = np.random.default_rng(2)
    A = rng.normal(size=(300, 3)).astype(np.float32) + 20
    B = rng.normal(size=(200, 3)).astype(np.float32) - 20
    X = np.concatenate([A, B])
    C0 = np.array([[5, 5, 5], [-5, -5, -5], [1000, 1000, 1000]], dtype=np.float32)
    C, a, counts, inertia = KM.lloyd_step(X, C0)
    np.testing.assert_allclose(C[0], A.astype(np.float64).mean(0), rtol=1e-12)
    np.testing.assert_allclose(C[1], B.astype(np.float64).mean(0), rtol=1e-12)
    np.testing.assert_array_equal(C[2], C0[2])            # empty cluster keeps its centre
    np.testing.assert_array_equal(counts, [300, 200, 0])
    ref = cdist(X.astype(np.float64), C0.astype(np.float64), "sqeuclidean").min(1).sum()
    assert abs(inertia - ref) <= 1e-5 * ref


def test_lloyd_inertia_is_monotone():
    rng = np.random.default_rng(3)
    X = rng.normal(size=(2000, 4)).astype(np.float32) * np.array([1, 3, 0.5, 2], np.float32)
    C0 = X[:8].copy()
    _, _, inertias = KM.kmeans(X, C0, 8)
    # each Lloyd iteration can only lower the objective (up to fp32 distance rounding)
    assert all(b <= a * (1 + 1e-6) for a, b in zip(inertias, inertias[1:]))


def test_seed_weights_scale():
    w = KM.seed_weights(np.array([0.0, 1.0, 3.0, 0.75], np.float32))
    # the largest distance (3.0) lands in [2^29, 2^30), ratios kept to 2^-29
    assert 2 ** 29 <= w.max() < 2 ** 30 and w[0] == 0
    np.testing.assert_allclose(w[1:] / w.max(), [1 / 3, 1, 0.25], rtol=2.0 ** -28)


def test_seeding_draw_follows_the_distance_law_exactly():
    """On a grid of M uniforms the number of draws landing on point i differs from
    M * w_i / total by at most one: the inverse-CDF step has no off-by-one."""
    X = np.array([[0.0], [1.0], [2.0], [4.0], [7.0]], dtype=np.float32)
    dist = KM.sqdist_fp32(X, X[:1])[:, 0]
    w = KM.seed_weights(dist)
    total = int(w.sum())
    M = 10007
    hits = np.zeros(5, dtype=np.int64)
    for j in range(M):
        u = (j + 0.5) / M
        _, C = KM.kmeanspp(X, 2, 0, [u])
        hits[int(np.flatnonzero(X[:, 0] == C[1, 0])[0])] += 1
    assert hits[0] == 0                                   # the chosen centre has weight 0
    assert np.all(np.abs(hits - M * w / total) <= 1.0)


def test_seeding_second_centre_is_the_far_point():
    X = np.array([[0, 0], [0, 0], [10, 0]], dtype=np.float32)
    for u in (0.0, 0.3, 0.999):
        idx, C = KM.kmeanspp(X, 2, 0, [u])
        assert idx[1] == 2 and np.array_equal(C[1], X[2])


def test_seeding_all_points_on_centres_repeats_the_last():
    X = np.ones((4, 3), dtype=np.float32)
    idx, _ = KM.kmeanspp(X, 3, 2, [0.5, 0.5])
    np.testing.assert_array_equal(idx, [2, 2, 2])
