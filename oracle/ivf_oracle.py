"""Plain CPU oracle for the IVF application of the soft assignment.

TEST INFRASTRUCTURE ONLY: imported by tests/ and bench.py's CPU legs, never by the
product path.  Shares no code with the CUDA library.

"Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", §4 (IVF
coarse quantizer): the index keeps, per cluster, the posting list of the vectors
assigned to it; with the multi-assignment of §4.3 a vector sits in the lists of its
top-2 clusters (r > tau).  A query probes the nprobe clusters whose centroids are
nearest, computes the exact distance to every vector of those lists ("distance
computations", DCO, counted per list entry scanned) and returns the k nearest.

Readings where the pages are silent (the same in the CUDA path):
  * list order: the vectors of a cluster in increasing index order;
  * distances: fp32 squared L2, dimensions in increasing order, every subtraction,
    product and sum rounded separately (as the k-means warm start), so that both sides
    rank identically; ties (equal distance) go to the lower index, for centroids and
    for vectors;
  * a vector met in several probed lists is returned once (DCO counts every scan);
  * fewer than k distinct candidates: the result is padded with id -1, distance +inf.
"""
from __future__ import annotations

import numpy as np

from oracle.kmeans_oracle import sqdist_fp32


def build(ids, K):
    """Posting lists from the soft-assignment ids [N, m] (-1 = none): (offsets [K+1],
    entries) with the entries of cluster k at offsets[k]:offsets[k+1], in increasing
    vector index."""
    ids = np.asarray(ids)
    N = ids.shape[0]
    lists = [[] for _ in range(K)]
    for i in range(N):
        for c in ids[i]:
            if c >= 0:
                lists[int(c)].append(i)
    offsets = np.zeros(K + 1, dtype=np.int64)
    offsets[1:] = np.cumsum([len(l) for l in lists])
    entries = np.array([i for l in lists for i in l], dtype=np.int64)
    return offsets, entries


def search(Q, centroids, offsets, entries, X, nprobe, k):
    """IVF search.  Returns (ids [nq, k] int64, dist [nq, k] fp32, dco [nq] int64)."""
    Q = np.asarray(Q, dtype=np.float32)
    C = np.asarray(centroids, dtype=np.float32)
    X = np.asarray(X, dtype=np.float32)
    nq = Q.shape[0]
    out_i = np.full((nq, k), -1, dtype=np.int64)
    out_d = np.full((nq, k), np.inf, dtype=np.float32)
    dco = np.zeros(nq, dtype=np.int64)
    dc = sqdist_fp32(Q, C)                                # [nq, K]
    for q in range(nq):
        order = sorted(range(C.shape[0]), key=lambda j: (dc[q, j], j))[:nprobe]
        cand = []
        for c in order:
            cand.extend(entries[offsets[c]:offsets[c + 1]].tolist())
        dco[q] = len(cand)
        uniq = sorted(set(cand))
        if not uniq:
            continue
        dv = sqdist_fp32(Q[q:q + 1], X[uniq])[0]
        best = sorted(zip(dv.tolist(), uniq))[:k]
        for r, (d, i) in enumerate(best):
            out_i[q, r] = i
            out_d[q, r] = d
    return out_i, out_d, dco
