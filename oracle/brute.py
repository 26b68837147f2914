"""Pure-Python brute-force EM step for tiny inputs (N <= ~64, K <= ~8, D <= ~4).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  A second, independent
statement of "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
Clustering", §2: scalar loops, math.fsum for every sum, math.exp / math.log for
the log-sum-exp, no NumPy.  It exists to catch a dropped term, a wrong sign or
a transposed index in gmm_oracle by disagreeing with it.
"""
from __future__ import annotations

import math

EMPTY_NK = 1e-6  # same reading as gmm_oracle, stated again on purpose


def log_density(x, mu, var, spherical):
    """log N(x | μ, Σ) for one point and one component (§2)."""
    D = len(x)
    if spherical:
        s = var  # scalar σ²
        return -0.5 * (D * math.log(2.0 * math.pi * s)
                       + math.fsum((x[d] - mu[d]) ** 2 for d in range(D)) / s)
    return -0.5 * math.fsum(math.log(2.0 * math.pi * var[d]) + (x[d] - mu[d]) ** 2 / var[d]
                            for d in range(D))


def em_step(X, w, mu, var, spherical=False, reg_covar=1e-6):
    """Returns (w_new, mu_new, var_new, loglik, logZ list, R list of lists)."""
    N, K, D = len(X), len(mu), len(X[0])
    logZ, R = [], []
    for i in range(N):
        lz = [(math.log(w[k]) if w[k] > 0 else -math.inf)
              + log_density(X[i], mu[k], var[k], spherical) for k in range(K)]
        m = max(lz)
        z = m + math.log(math.fsum(math.exp(v - m) for v in lz))
        logZ.append(z)
        R.append([math.exp(v - z) for v in lz])
    loglik = math.fsum(logZ)
    Nk = [math.fsum(R[i][k] for i in range(N)) for k in range(K)]
    live = [Nk[k] >= EMPTY_NK for k in range(K)]
    tot = math.fsum(Nk[k] for k in range(K) if live[k])
    w_new, mu_new, var_new = [], [], []
    for k in range(K):
        if not live[k]:
            w_new.append(0.0)
            mu_new.append(list(mu[k]))
            var_new.append(var[k] if spherical else list(var[k]))
            continue
        w_new.append(Nk[k] / tot)
        m_k = [math.fsum(R[i][k] * X[i][d] for i in range(N)) / Nk[k] for d in range(D)]
        mu_new.append(m_k)
        per_d = [math.fsum(R[i][k] * (X[i][d] - m_k[d]) ** 2 for i in range(N)) / Nk[k]
                 for d in range(D)]
        if spherical:
            var_new.append(math.fsum(per_d) / D + reg_covar)
        else:
            var_new.append([v + reg_covar for v in per_d])
    return w_new, mu_new, var_new, loglik, logZ, R


def top_m_assign(X, w, mu, var, top_m, r_threshold, spherical=False):
    """Brute-force §4.3 multi-assignment: full sort of each row, ties by index."""
    N, K = len(X), len(mu)
    ids, resp = [], []
    for i in range(N):
        lz = [(math.log(w[k]) if w[k] > 0 else -math.inf)
              + log_density(X[i], mu[k], var[k], spherical) for k in range(K)]
        m = max(lz)
        z = m + math.log(math.fsum(math.exp(v - m) for v in lz))
        order = sorted(range(K), key=lambda k: (-lz[k], k))
        row_i, row_r = [], []
        for rank in range(top_m):
            k = order[rank] if rank < K else None
            r = math.exp(lz[k] - z) if k is not None else 0.0
            if k is not None and (rank == 0 or r > r_threshold):
                row_i.append(k)
                row_r.append(r)
            else:
                row_i.append(-1)
                row_r.append(0.0)
        ids.append(row_i)
        resp.append(row_r)
    return ids, resp


def shard_statistics(X, w, mu, var, spherical=False):
    """Per component [N_k, Σ r (x_d − μ_kd) for each d, Σ r (x_d − μ_kd)² for each d]
    about the input means, flattened, then Σ log Z (scalar loops, math.fsum)."""
    N, K, D = len(X), len(mu), len(X[0])
    *_, logZ, R = em_step(X, w, mu, var, spherical)
    out = []
    for k in range(K):
        out.append(math.fsum(R[i][k] for i in range(N)))
        out.extend(math.fsum(R[i][k] * (X[i][d] - mu[k][d]) for i in range(N)) for d in range(D))
        out.extend(math.fsum(R[i][k] * (X[i][d] - mu[k][d]) ** 2 for i in range(N))
                   for d in range(D))
    out.append(math.fsum(logZ))
    return out


def fisher_vector(X, w, mu, var, spherical=False):
    """Fisher vector [G_mu, G_sigma] by scalar loops (same definition as the NumPy oracle)."""
    N, K, D = len(X), len(mu), len(X[0])
    *_, R = em_step(X, w, mu, var, spherical)
    gm, gs = [], []
    for k in range(K):
        for d in range(D):
            sd = math.sqrt(var[k] if spherical else var[k][d])
            gm.append(math.fsum(R[i][k] * (X[i][d] - mu[k][d]) / sd for i in range(N))
                      / (N * math.sqrt(w[k])))
    for k in range(K):
        for d in range(D):
            sd = math.sqrt(var[k] if spherical else var[k][d])
            gs.append(math.fsum(R[i][k] * (((X[i][d] - mu[k][d]) / sd) ** 2 - 1.0)
                                for i in range(N)) / (N * math.sqrt(2.0 * w[k])))
    return gm + gs
