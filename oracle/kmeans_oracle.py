"""Plain CPU oracle for the k-means warm start that precedes EM.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and bench.py's
CPU legs, never by the product path.  Shares no code with the CUDA library.

"Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering" initialises the
mixture from k-means (§4.4: k-means, then soft EM from the resulting centroids; the
appendix on initialisation: a k-means warm start, or k-means++ seeding).  What is
computed here:

  seeding (k-means++, Arthur & Vassilvitskii 2007)
      c_0 = x_{first};  for t = 1 .. K-1:  D(x) = min_{j < t} ||x - c_j||^2,
      c_t = x_i with probability D(x_i) / sum_i D(x_i)
  Lloyd iteration
      a_i = argmin_k ||x_i - c_k||^2            (ties: lower k)
      c_k = mean of {x_i : a_i = k}             (empty cluster: c_k kept)
      inertia = sum_i ||x_i - c_{a_i}||^2

Readings where the pages are silent (stated again in the product's documentation):
  * The random draws of the seeding are inputs: the index of the first centre and one
    uniform u_t in [0, 1) per later centre.
  * Decisions that floating point makes into integers (the argmin, the seeding draw) are
    taken in the precision the CUDA kernels use, so that both sides choose the same
    index: squared distances are fp32, accumulated over dimensions in increasing order,
    each subtraction, product and sum rounded separately (no fused multiply-add).  The
    seeding weights are those fp32 distances turned into integers,
    w_i = floor(D(x_i) * 2^s) with 2^s the power of two that brings the largest D to
    [2^29, 2^30); the draw picks the smallest i whose running integer sum exceeds
    floor(u_t * total) (u_t * total rounded once in fp64).
  * Centroids and inertia are fp64 sums of the fp32 data (so they agree with the
    kernels up to summation order).
"""
from __future__ import annotations

import numpy as np


def sqdist_fp32(X, C):
    """[N, K] squared distances in fp32, dimension by dimension in increasing order,
    every operation rounded to fp32 separately."""
    X = np.asarray(X, dtype=np.float32)
    C = np.asarray(C, dtype=np.float32)
    N, D = X.shape
    K = C.shape[0]
    acc = np.zeros((N, K), dtype=np.float32)
    for d in range(D):
        t = np.subtract(X[:, d][:, None], C[:, d][None, :], dtype=np.float32)
        sq = np.multiply(t, t, dtype=np.float32)
        acc = np.add(acc, sq, dtype=np.float32)
    return acc


def assign(X, C):
    """Lloyd assignment step: (a_i, d_i) with a_i = argmin_k, lowest k on ties."""
    Dm = sqdist_fp32(X, C)
    a = np.argmin(Dm, axis=1).astype(np.int32)        # numpy returns the first minimum
    return a, Dm[np.arange(Dm.shape[0]), a]


def lloyd_step(X, C):
    """One Lloyd iteration.  Returns (new centroids fp64, assignments, counts, inertia)."""
    X = np.asarray(X, dtype=np.float32)
    C = np.asarray(C)
    K, D = C.shape
    a, dmin = assign(X, C)
    counts = np.bincount(a, minlength=K).astype(np.int64)
    sums = np.zeros((K, D), dtype=np.float64)
    np.add.at(sums, a, X.astype(np.float64))
    Cn = np.array(C, dtype=np.float64, copy=True)
    live = counts > 0
    Cn[live] = sums[live] / counts[live, None]
    inertia = float(np.sum(dmin.astype(np.float64)))
    return Cn, a, counts, inertia


def seed_weights(dist):
    """Integer seeding weights from fp32 squared distances (see the module docstring)."""
    dist = np.asarray(dist, dtype=np.float32)
    mx = float(dist.max()) if dist.size else 0.0
    if not mx > 0.0:
        return np.zeros(dist.shape, dtype=np.int64)
    e = int(np.frexp(mx)[1])                 # mx in [2^(e-1), 2^e)
    scale = np.ldexp(1.0, 30 - e)            # mx * scale in [2^29, 2^30)
    return np.floor(dist.astype(np.float64) * scale).astype(np.int64)


def kmeanspp(X, K, first, u):
    """k-means++ seeding with the given first index and uniforms u[0 .. K-2].
    Returns (indices of the chosen points, centroids fp32)."""
    X = np.asarray(X, dtype=np.float32)
    N = X.shape[0]
    idx = [int(first)]
    dist = sqdist_fp32(X, X[first:first + 1])[:, 0]
    for t in range(1, K):
        w = seed_weights(dist)
        total = int(w.sum())
        if total == 0:                        # every point sits on a chosen centre
            i = idx[-1]
        else:
            target = int(np.floor(float(u[t - 1]) * float(total)))
            csum = np.cumsum(w)
            i = int(np.searchsorted(csum, target, side="right"))
            i = min(i, N - 1)
        idx.append(i)
        dist = np.minimum(dist, sqdist_fp32(X, X[i:i + 1])[:, 0])
    return np.array(idx, dtype=np.int64), X[idx].copy()


def kmeans(X, C0, iters):
    """`iters` Lloyd iterations from C0.  Returns (centroids, assignments, inertias)."""
    C = np.asarray(C0, dtype=np.float32)
    inertias = []
    a = None
    for _ in range(iters):
        Cn, a, _, inertia = lloyd_step(X, C)
        inertias.append(inertia)
        C = Cn.astype(np.float32)
    return C, a, inertias
