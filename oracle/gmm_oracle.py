"""Plain, slow, fp64 NumPy oracle for one EM iteration of a Gaussian mixture.

TEST INFRASTRUCTURE ONLY: imported by tests/, __graft_entry__.smoke() and the
CPU-baseline leg of bench.py, never by the product path.  Shares no code with
the CUDA library.

Follows "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering",
§2 (Gaussian Mixture Models) equation by equation:

  density        p(x | Θ) = Σ_k π_k N(x | μ_k, Σ_k)          (§2, mixture density)
  log-likelihood log p(X | Θ) = Σ_i log Σ_k π_k N_ik           (§2)
  E-step         z_ik = π_k N_ik,  r_ik = z_ik / Σ_j z_ij      (§2), in log space
                 with a max-shifted log-sum-exp (§2, numerical stability)
  M-step         N_k = Σ_i r_ik,  π_k = N_k / N                (§2, Eq. (1))
                 μ_k = (1/N_k) Σ_i r_ik x_i                    (§2, Eq. (2))
                 σ_k² = (1/(D N_k)) Σ_i r_ik ‖x_i − μ_k‖²      (§2, Eq. (3)),
                 with the *updated* mean ("followed by an updated variance").
  stopping       small change of the log-likelihood, or a maximum number of
                 iterations (§2, last paragraph).
  assignment     argmax responsibility (§4.2) and top-2 with r_ik > τ (§4.3).

The paper's model is isotropic, Σ_k = σ_k² I (§2 footnote 1; Appendix A).  The
diagonal model Σ_k = diag(σ_k1², …, σ_kD²) is the same equations applied per
dimension: Eq. (3) without the 1/D average.  Both are implemented here.

Readings where the paper is silent (each stated where it is used):
  * π_k = N_k / Σ_k' N_k' (Algorithm 1, last step) instead of N_k / N (Eq. (1));
    equal in exact arithmetic, the former keeps Σ π = 1 under rounding.
  * variance floor: σ² ← σ²_ML + reg_covar (additive, default 1e-6).
  * empty component (N_k < EMPTY_NK): its mean and variance are kept and its
    weight becomes exactly 0 (log π = −inf, so it stays out afterwards).  If
    every component is empty the step is an error.
  * soft assignment ranks components by their log joint (ties: lower index),
    always keeps rank 1, keeps ranks 2..m only where r > r_threshold (strict),
    and pads with id −1, r 0.

The log-density is evaluated in the direct (x − μ)² form, not the expanded
dot-product form the tensor-core kernel uses, so the two do not share a
rounding pattern.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

COV_DIAG = 0
COV_SPHERICAL = 1

# A component whose total responsibility mass is below this many effective
# points is treated as empty (see module docstring).
EMPTY_NK = 1e-6

# RAM budget for one dense row chunk of the N x K log-density matrix.
_CHUNK_BYTES = 512 << 20


def _as_f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _row_chunks(n: int, k: int):
    step = max(1, _CHUNK_BYTES // (8 * max(k, 1) * 3))
    for s in range(0, n, step):
        yield s, min(n, s + step)


def _cache_blocks(n: int, d: int):
    step = max(1, (256 << 10) // (8 * max(d, 1)))   # ~256 KB row blocks
    for s in range(0, n, step):
        yield s, min(n, s + step)


def log_gauss(X, means, variances, cov_type=COV_DIAG):
    """Dense log N(x_i | μ_k, Σ_k), shape [N, K], in the direct (x − μ)² form.

    §2: N(x | μ_k, σ_k² I) for the isotropic model; per-dimension σ_kd² for the
    diagonal model.  log N = −½ Σ_d [log(2π σ_kd²) + (x_d − μ_kd)² / σ_kd²].
    """
    X = _as_f64(X)
    means = _as_f64(means)
    variances = _as_f64(variances)
    N, D = X.shape
    K = means.shape[0]
    out = np.empty((N, K), dtype=np.float64)
    if cov_type == COV_DIAG:
        var = variances.reshape(K, D)
        norm = -0.5 * np.sum(np.log(2.0 * math.pi * var), axis=1)  # [K]
        prec = 1.0 / var
        for s, e in _cache_blocks(N, D):
            diff = np.empty_like(X[s:e])
            for k in range(K):
                np.subtract(X[s:e], means[k], out=diff)
                diff *= diff                                    # (x_d − μ_kd)²
                out[s:e, k] = norm[k] - 0.5 * (diff @ prec[k])  # Σ_d (x_d − μ_kd)² / σ_kd²
    elif cov_type == COV_SPHERICAL:
        var = variances.reshape(K)
        norm = -0.5 * D * np.log(2.0 * math.pi * var)
        for s, e in _cache_blocks(N, D):
            diff = np.empty_like(X[s:e])
            for k in range(K):
                np.subtract(X[s:e], means[k], out=diff)
                diff *= diff
                out[s:e, k] = norm[k] - 0.5 * np.sum(diff, axis=1) / var[k]
    else:
        raise ValueError("cov_type")
    return out


def log_joint(X, weights, means, variances, cov_type=COV_DIAG):
    """log z_ik = log π_k + log N(x_i | θ_k)  (§2, unnormalised score)."""
    w = _as_f64(weights)
    with np.errstate(divide="ignore"):
        logw = np.log(w)
    return log_gauss(X, means, variances, cov_type) + logw[None, :]


def logsumexp_rows(L):
    """log Σ_k exp(L_ik), max-shifted (§2, log-sum-exp); rows of −inf give −inf."""
    m = np.max(L, axis=1)
    safe = np.where(np.isfinite(m), m, 0.0)
    with np.errstate(divide="ignore"):
        s = np.log(np.sum(np.exp(L - safe[:, None]), axis=1))
    return safe + s


def e_step(X, weights, means, variances, cov_type=COV_DIAG):
    """E-step of §2: per-point log Z_i and the dense responsibilities R[N, K]."""
    L = log_joint(X, weights, means, variances, cov_type)
    logZ = logsumexp_rows(L)
    R = np.exp(L - logZ[:, None])
    return logZ, R


@dataclass
class StepResult:
    weights: np.ndarray
    means: np.ndarray
    variances: np.ndarray
    loglik: float          # log p(X | Θ_in): the likelihood of the INPUT parameters
    logZ: np.ndarray       # per-point log p(x_i | Θ_in)
    Nk: np.ndarray         # effective counts N_k (Eq. (1))
    empty: np.ndarray      # bool[K], components treated as empty


def em_step(X, weights, means, variances, cov_type=COV_DIAG, reg_covar=1e-6):
    """One EM iteration: E-step then M-step Eqs. (1)-(3), §2.

    The dense R is formed chunk by chunk over rows; the mean needs a full pass
    before the variance (Eq. (3) uses the updated mean), so R is recomputed in
    a second pass when it does not fit one chunk.
    """
    X = _as_f64(X)
    N, D = X.shape
    means_in = _as_f64(means)
    K = means_in.shape[0]
    var_in = _as_f64(variances)
    w_in = _as_f64(weights)

    # Pass A: log Z, N_k = Σ r (Eq. (1)), Σ r x (numerator of Eq. (2)).
    logZ = np.empty(N, dtype=np.float64)
    Nk = np.zeros(K, dtype=np.float64)
    Sx = np.zeros((K, D), dtype=np.float64)
    for s, e in _row_chunks(N, K):
        lz, R = e_step(X[s:e], w_in, means_in, var_in, cov_type)
        logZ[s:e] = lz
        Nk += R.sum(axis=0)
        Sx += R.T @ X[s:e]
    loglik = float(np.sum(logZ))
    if not np.all(np.isfinite(logZ)):
        # every weight zero, or a point with zero density under every component
        raise FloatingPointError("non-finite log-likelihood")

    empty = Nk < EMPTY_NK
    if np.all(empty):
        raise FloatingPointError("every component is empty")
    live = ~empty
    mu_new = means_in.copy()
    mu_new[live] = Sx[live] / Nk[live, None]                       # Eq. (2)

    # Pass B: Σ r ‖x − μ_new‖² (Eq. (3)), per dimension for the diagonal model.
    Sq = np.zeros((K, D), dtype=np.float64)
    chunks = list(_row_chunks(N, K))
    for s, e in chunks:
        if len(chunks) > 1:
            _, R = e_step(X[s:e], w_in, means_in, var_in, cov_type)
        for bs, be in _cache_blocks(e - s, D):
            Xb = X[s + bs:s + be]
            diff = np.empty_like(Xb)
            for k in np.nonzero(live)[0]:
                np.subtract(Xb, mu_new[k], out=diff)
                diff *= diff
                Sq[k] += R[bs:be, k] @ diff                # Σ_i r_ik (x_id − μ_kd)²
    if cov_type == COV_DIAG:
        var_new = var_in.reshape(K, D).copy()
        var_new[live] = Sq[live] / Nk[live, None] + reg_covar       # Eq. (3), per d
    else:
        var_new = var_in.reshape(K).copy()
        var_new[live] = Sq[live].sum(axis=1) / (D * Nk[live]) + reg_covar  # Eq. (3)

    w_new = np.zeros(K, dtype=np.float64)
    w_new[live] = Nk[live] / np.sum(Nk[live])                      # Eq. (1)
    return StepResult(w_new, mu_new, var_new, loglik, logZ, Nk, empty)


def shard_statistics(X, weights, means, variances, cov_type=COV_DIAG, logz_out=None):
    """The sufficient statistics one shard of the rows contributes to an EM step.

    Layout (fp64, length K (1 + 2D) + 1), per component k at offset k (1 + 2D):
      N_k = Σ_i r_ik,   Σ_i r_ik (x_id − μ_kd),   Σ_i r_ik (x_id − μ_kd)²   (d < D)
    about the INPUT means μ_k, then Σ_i log Z_i.  Every entry is a sum over rows, so
    the statistics of disjoint shards add up to those of their union; §2's M-step
    (Eqs. (1)-(3)) is a function of the sums alone (m_step_from_statistics).
    logz_out: optional float64 array [N] that receives the per-point log Z_i.
    """
    X = _as_f64(X)
    N, D = X.shape
    mu = _as_f64(means)
    K = mu.shape[0]
    row = 1 + 2 * D
    out = np.zeros(K * row + 1, dtype=np.float64)
    st = out[:K * row].reshape(K, row)
    ll = 0.0
    for s, e in _row_chunks(N, K):
        lz, R = e_step(X[s:e], weights, mu, variances, cov_type)
        if logz_out is not None:
            logz_out[s:e] = lz
        ll += float(np.sum(lz))
        st[:, 0] += R.sum(axis=0)
        for k in range(K):
            diff = X[s:e] - mu[k]
            st[k, 1:1 + D] += R[:, k] @ diff
            st[k, 1 + D:] += R[:, k] @ (diff * diff)
    out[K * row] = ll
    return out


def m_step_from_statistics(stats, weights, means, variances, cov_type=COV_DIAG,
                           reg_covar=1e-6):
    """§2's M-step from summed shard statistics (layout of shard_statistics).

    With S1 = Σ r (x − μ) and S2 = Σ r (x − μ)² about the input mean μ:
      μ_new = μ + S1 / N_k                                           (Eq. (2))
      Σ r (x − μ_new)² = S2 − S1² / N_k, so σ² = S2 / N_k − (S1 / N_k)²  (Eq. (3))
    plus the same readings as em_step (weights over live components, additive floor,
    empty components kept).  Returns a StepResult with logZ = None.
    """
    stats = _as_f64(stats)
    mu_in = _as_f64(means)
    K, D = mu_in.shape
    row = 1 + 2 * D
    st = stats[:K * row].reshape(K, row)
    loglik = float(stats[K * row])
    if not np.isfinite(loglik):
        raise FloatingPointError("non-finite log-likelihood")
    Nk = st[:, 0].copy()
    empty = Nk < EMPTY_NK
    if np.all(empty):
        raise FloatingPointError("every component is empty")
    live = ~empty
    m1 = np.zeros((K, D))
    m1[live] = st[live, 1:1 + D] / Nk[live, None]
    v = np.zeros((K, D))
    v[live] = np.maximum(st[live, 1 + D:] / Nk[live, None] - m1[live] ** 2, 0.0)
    mu_new = mu_in.copy()
    mu_new[live] = mu_in[live] + m1[live]
    var_in = _as_f64(variances)
    if cov_type == COV_DIAG:
        var_new = var_in.reshape(K, D).copy()
        var_new[live] = v[live] + reg_covar
    else:
        var_new = var_in.reshape(K).copy()
        var_new[live] = v[live].mean(axis=1) + reg_covar
    w_new = np.zeros(K)
    w_new[live] = Nk[live] / np.sum(Nk[live])
    return StepResult(w_new, mu_new, var_new, loglik, None, Nk, empty)


def fisher_vector(X, weights, means, variances, cov_type=COV_DIAG, normalize=False):
    """Fisher-vector encoding of the set X under the mixture (gradients of the average
    log-likelihood with respect to the means and standard deviations, whitened by the
    diagonal Fisher information: Perronnin & Dance 2007; Sanchez et al. 2013).  The
    paper names the encoding as a use of the same fused E-step and weighted statistics
    (§6) without defining it; this is the textbook definition:

      G_mu_kd    = 1 / (N sqrt(pi_k))   sum_i r_ik (x_id - mu_kd) / sigma_kd
      G_sigma_kd = 1 / (N sqrt(2 pi_k)) sum_i r_ik ((x_id - mu_kd)^2 / sigma_kd^2 - 1)

    returned as [G_mu (K x D, row-major), G_sigma (K x D)] (length 2 K D).  With
    normalize, the "improved" encoding: z <- sign(z) sqrt(|z|), then z / ||z||_2.
    Components with pi_k = 0 contribute zeros.
    """
    X = _as_f64(X)
    N, D = X.shape
    mu = _as_f64(means)
    K = mu.shape[0]
    w = _as_f64(weights)
    var = _as_f64(variances)
    sig = np.sqrt(var.reshape(K, 1) * np.ones((1, D)) if cov_type == COV_SPHERICAL
                  else var.reshape(K, D))
    gm = np.zeros((K, D))
    gs = np.zeros((K, D))
    for s, e in _row_chunks(N, K):
        _, R = e_step(X[s:e], w, mu, var, cov_type)
        for k in range(K):
            z = (X[s:e] - mu[k]) / sig[k]
            gm[k] += R[:, k] @ z
            gs[k] += R[:, k] @ (z * z - 1.0)
    live = w > 0
    gm[live] /= (N * np.sqrt(w[live]))[:, None]
    gs[live] /= (N * np.sqrt(2.0 * w[live]))[:, None]
    gm[~live] = 0.0
    gs[~live] = 0.0
    fv = np.concatenate([gm.ravel(), gs.ravel()])
    if normalize:
        fv = np.sign(fv) * np.sqrt(np.abs(fv))
        nrm = np.linalg.norm(fv)
        if nrm > 0:
            fv = fv / nrm
    return fv


def fit(X, weights, means, variances, cov_type=COV_DIAG, reg_covar=1e-6,
        max_iters=100, tol=0.0):
    """Repeat em_step; stop after max_iters or when |L_t − L_{t−1}| / N < tol.

    §2, last paragraph: "a sufficiently small change in the log-likelihood
    between successive iterations or ... a predefined maximum number of
    iterations".  The per-point normalisation of the change is a reading.
    Returns (weights, means, variances, logliks[list], iters_done).
    """
    X = _as_f64(X)
    N = X.shape[0]
    w, mu, var = _as_f64(weights), _as_f64(means), _as_f64(variances)
    lls = []
    it = 0
    for it in range(1, max_iters + 1):
        r = em_step(X, w, mu, var, cov_type, reg_covar)
        w, mu, var = r.weights, r.means, r.variances
        lls.append(r.loglik)
        if tol > 0 and len(lls) >= 2 and abs(lls[-1] - lls[-2]) / N < tol:
            break
    return w, mu, var, lls, it


def soft_assign(X, weights, means, variances, cov_type=COV_DIAG, top_m=2,
                r_threshold=0.0):
    """Multi-assignment from responsibilities (§4.2 argmax, §4.3 top-2 > τ).

    Components are ranked by log z_ik (monotone in r_ik), ties to the lower
    index.  Rank 1 is always kept (§4.2: every vector lands in its most
    responsible cluster); ranks 2..top_m are kept only where r_ik > r_threshold.
    Returns ids int32[N, top_m] (−1 padded) and resp float64[N, top_m] (0 padded).
    """
    X = _as_f64(X)
    N = X.shape[0]
    ids = np.full((N, top_m), -1, dtype=np.int32)
    resp = np.zeros((N, top_m), dtype=np.float64)
    K = _as_f64(means).shape[0]
    for s, e in _row_chunks(N, K):
        L = log_joint(X[s:e], weights, means, variances, cov_type)
        logZ = logsumexp_rows(L)
        # stable sort on −L: equal keys keep ascending component order
        order = np.argsort(-L, axis=1, kind="stable")[:, :top_m]
        top_l = np.take_along_axis(L, order, axis=1)
        top_r = np.exp(top_l - logZ[:, None])
        keep = np.zeros_like(top_r, dtype=bool)
        keep[:, 0] = True
        keep[:, 1:] = top_r[:, 1:] > r_threshold
        ids[s:e] = np.where(keep, order, -1).astype(np.int32)
        resp[s:e] = np.where(keep, top_r, 0.0)
    return ids, resp
