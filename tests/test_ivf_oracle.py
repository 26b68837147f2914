"""Pins of the IVF oracle (oracle/ivf_oracle.py): a hand-built index, exhaustive
probing equals brute-force k-NN, duplicates from multi-assignment, padding."""
import numpy as np

from oracle import ivf_oracle as IVF
from oracle import kmeans_oracle as KM


def test_build_by_hand():
    ids = np.array([[2, -1], [0, 2], [2, 1], [1, -1]])
    off, ent = IVF.build(ids, 3)
    np.testing.assert_array_equal(off, [0, 1, 3, 6])
    np.testing.assert_array_equal(ent, [1, 2, 3, 0, 1, 2])


def test_exhaustive_probe_is_brute_force_knn():
    rng = np.random.default_rng(0)
    X = rng.normal(size=(400, 6)).astype(np.float32)
    Q = rng.normal(size=(25, 6)).astype(np.float32)
    C = X[:10].copy()
    a, _ = KM.assign(X, C)
    off, ent = IVF.build(a[:, None], 10)
    ids, dist, dco = IVF.search(Q, C, off, ent, X, nprobe=10, k=7)
    # independent brute force in fp64 (no ties in continuous data)
    d64 = ((Q[:, None, :].astype(np.float64) - X[None].astype(np.float64)) ** 2).sum(-1)
    np.testing.assert_array_equal(ids, np.argsort(d64, axis=1)[:, :7])
    assert np.all(dco == 400)
    np.testing.assert_allclose(dist, np.sort(d64, axis=1)[:, :7], rtol=1e-5)


def test_duplicates_are_returned_once_and_counted_twice():
    X = np.array([[0, 0], [1, 0], [5, 5]], dtype=np.float32)
    C = np.array([[0, 0], [1, 1]], dtype=np.float32)
    ids = np.array([[0, 1], [0, -1], [1, -1]])              # vector 0 in both lists
    off, ent = IVF.build(ids, 2)
    out, dist, dco = IVF.search(np.array([[0.1, 0.0]], np.float32), C, off, ent, X, 2, 4)
    assert dco[0] == 4
    np.testing.assert_array_equal(out[0], [0, 1, 2, -1])
    assert np.isinf(dist[0, 3])


def test_single_probe_sees_only_its_list():
    X = np.array([[0, 0], [10, 10], [0.5, 0]], dtype=np.float32)
    C = np.array([[0, 0], [10, 10]], dtype=np.float32)
    off, ent = IVF.build(np.array([[0], [1], [0]]), 2)
    out, _, dco = IVF.search(np.array([[9, 9]], np.float32), C, off, ent, X, 1, 2)
    np.testing.assert_array_equal(out[0], [1, -1])
    assert dco[0] == 1
