"""Teacher-forced oracle steps on inputs too large for one core: the rows are split
into shards, a pool of worker processes (started with "spawn", so that no worker
inherits a CUDA context) runs the oracle's shard_statistics on each, the shard
vectors are added in shard order, and the oracle's m_step_from_statistics gives the
step.  Every number comes from oracle/ (test infrastructure; the CUDA library is not
involved).  The shard split does not change the result beyond fp64 rounding: the
statistics are sums over rows (pinned by the oracle's additivity test)."""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def _shard(args):
    X, w, mu, var, cov = args
    from oracle import gmm_oracle as O
    lz = np.empty(X.shape[0], dtype=np.float64)
    st = O.shard_statistics(X, w, mu, var, cov, logz_out=lz)
    return st, lz


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def teacher_forced_step(X, weights, means, variances, cov=0, reg=1e-6, procs=None,
                        rows_per_shard=16384):
    """One oracle EM step from the given parameters, over all rows of X (fp64 numpy or
    anything np.asarray takes).  Returns the oracle's StepResult with logZ filled in."""
    from oracle import gmm_oracle as O
    X = np.asarray(X, np.float64)
    w = np.asarray(weights, np.float64)
    mu = np.asarray(means, np.float64)
    var = np.asarray(variances, np.float64)
    n = X.shape[0]
    bounds = list(range(0, n, rows_per_shard)) + [n]
    jobs = [(X[a:b], w, mu, var, cov) for a, b in zip(bounds[:-1], bounds[1:])]
    procs = max(1, min(procs or host_cores(), 32, len(jobs)))
    if procs == 1:
        parts = [_shard(j) for j in jobs]
    else:
        with mp.get_context("spawn").Pool(procs) as pool:
            parts = pool.map(_shard, jobs, chunksize=1)
    st = np.zeros_like(parts[0][0])
    for p, _ in parts:
        st += p
    res = O.m_step_from_statistics(st, w, mu, var, cov, reg)
    res.logZ = np.concatenate([lz for _, lz in parts])
    return res


def teacher_forced_step_stream(rows, n, weights, means, variances, cov=0, reg=1e-6,
                               procs=None, rows_per_shard=16384):
    """teacher_forced_step for an X that is not held on the host as a whole: rows(a, b)
    returns rows a .. b-1 as an fp64 numpy array (for example copied from the device), and
    the shards are produced while the pool works on earlier ones."""
    from oracle import gmm_oracle as O
    w = np.asarray(weights, np.float64)
    mu = np.asarray(means, np.float64)
    var = np.asarray(variances, np.float64)
    bounds = list(range(0, n, rows_per_shard)) + [n]

    def jobs():
        for a, b in zip(bounds[:-1], bounds[1:]):
            yield (rows(a, b), w, mu, var, cov)

    procs = max(1, min(procs or host_cores(), 64))
    st = None
    lzs = []
    with mp.get_context("spawn").Pool(procs) as pool:
        for p, lz in pool.imap(_shard, jobs(), chunksize=1):   # in shard order
            st = p.copy() if st is None else st + p
            lzs.append(lz)
    res = O.m_step_from_statistics(st, w, mu, var, cov, reg)
    res.logZ = np.concatenate(lzs)
    return res
