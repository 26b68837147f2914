"""Teacher-forced oracle steps on inputs too large for one core: the rows are split
into shards, a pool of worker processes (started with "spawn", so that no worker
inherits a CUDA context) runs the oracle's shard_statistics on each, the shard
vectors are added in shard order, and the oracle's m_step_from_statistics gives the
step.  Every number comes from oracle/ (test infrastructure; the CUDA library is not
involved).  The shard split does not change the result beyond fp64 rounding: the
statistics are sums over rows (pinned by the oracle's additivity test).

Shards are small (2048 rows) so that the oracle's per-component temporaries stay in
cache; each worker receives the parameters once and uses one BLAS thread."""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

ROWS = 2048
_params = None


def _init(w, mu, var, cov):
    global _params
    _params = (w, mu, var, cov)
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass


def _shard(X):
    from oracle import gmm_oracle as O
    w, mu, var, cov = _params
    lz = np.empty(X.shape[0], dtype=np.float64)
    st = O.shard_statistics(X, w, mu, var, cov, logz_out=lz)
    return st, lz


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _run(shards, n_jobs, w, mu, var, cov, reg, procs):
    from oracle import gmm_oracle as O
    procs = max(1, min(procs or host_cores(), 64, n_jobs))
    st = None
    lzs = []
    if procs == 1:
        _init(w, mu, var, cov)
        results = map(_shard, shards)
        pool = None
    else:
        pool = mp.get_context("spawn").Pool(procs, initializer=_init, initargs=(w, mu, var, cov))
        results = pool.imap(_shard, shards, chunksize=4)     # in shard order
    try:
        for p, lz in results:
            st = p.copy() if st is None else st + p
            lzs.append(lz)
    finally:
        if pool is not None:
            pool.close()
            pool.join()
    res = O.m_step_from_statistics(st, w, mu, var, cov, reg)
    res.logZ = np.concatenate(lzs)
    return res


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, np.float64))


def teacher_forced_step(X, weights, means, variances, cov=0, reg=1e-6, procs=None):
    """One oracle EM step from the given parameters, over all rows of X (fp64 numpy or
    anything np.asarray takes).  Returns the oracle's StepResult with logZ filled in."""
    X = _f64(X)
    n = X.shape[0]
    shards = (X[a:a + ROWS] for a in range(0, n, ROWS))
    return _run(shards, -(-n // ROWS), _f64(weights), _f64(means), _f64(variances), cov, reg,
                procs)


def teacher_forced_step_stream(rows, n, weights, means, variances, cov=0, reg=1e-6,
                               procs=None, block=1 << 20):
    """teacher_forced_step for an X that is not held on the host as a whole: rows(a, b)
    returns rows a .. b-1 as an fp64 numpy array (for example copied from the device) and
    is called for blocks of `block` rows while the pool works on earlier shards."""
    def shards():
        for a in range(0, n, block):
            Xb = _f64(rows(a, min(n, a + block)))
            for s in range(0, Xb.shape[0], ROWS):
                yield Xb[s:s + ROWS]
    return _run(shards(), -(-n // ROWS), _f64(weights), _f64(means), _f64(variances), cov, reg,
                procs)
