"""Pins for the fp64 oracle against things other than itself.

Each test ties a part of oracle/gmm_oracle.py to the paper's definitions
("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", §2 and
§4.2-4.3) through a closed form, a library routine that computes the same
special case, an invariant, or an independent brute-force statement.  A
plausible mistake (a dropped term, a sign, a transposed operand, the old mean
in Eq. (3), π normalised wrongly) fails at least one of them.
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats
from scipy.spatial.distance import cdist

from oracle import brute
from oracle import gmm_oracle as O


def _rand_problem(rng, N, K, D, spherical=False, spread=3.0):
    X = rng.normal(size=(N, D)) * spread
    mu = X[rng.choice(N, K, replace=False)] + rng.normal(size=(K, D)) * 0.1
    w = rng.uniform(0.2, 1.0, size=K)
    w /= w.sum()
    var = rng.uniform(0.3, 4.0, size=K) if spherical else rng.uniform(0.3, 4.0, size=(K, D))
    return X, w, mu, var


# ----------------------------------------------------------------- K = 1 closed form
@pytest.mark.parametrize("cov", [O.COV_DIAG, O.COV_SPHERICAL])
def test_k1_closed_form(cov):
    """§2 Eqs. (1)-(3) with r ≡ 1: π = 1, μ = sample mean, σ² = population
    variance (÷N), averaged over d for the isotropic model; log Z is the plain
    Gaussian log-density (scipy.stats.norm.logpdf summed over d)."""
    rng = np.random.default_rng(1)
    N, D = 257, 5
    X = rng.normal(loc=[1.0, -2.0, 0.5, 3.0, 0.0], scale=[0.5, 2.0, 1.0, 3.0, 0.1], size=(N, D))
    mu0 = np.zeros((1, D))
    var0 = np.array([2.0]) if cov == O.COV_SPHERICAL else np.full((1, D), 2.0)
    reg = 1e-3
    r = O.em_step(X, [1.0], mu0, var0, cov, reg)
    assert r.weights[0] == pytest.approx(1.0, abs=1e-15)
    np.testing.assert_allclose(r.means[0], X.mean(axis=0), rtol=1e-13, atol=1e-13)
    pop_var = X.var(axis=0, ddof=0)
    if cov == O.COV_DIAG:
        np.testing.assert_allclose(r.variances[0], pop_var + reg, rtol=1e-12)
        lz = scipy.stats.norm.logpdf(X, loc=0.0, scale=np.sqrt(2.0)).sum(axis=1)
    else:
        assert r.variances[0] == pytest.approx(pop_var.mean() + reg, rel=1e-12)
        lz = scipy.stats.norm.logpdf(X, loc=0.0, scale=np.sqrt(2.0)).sum(axis=1)
    np.testing.assert_allclose(r.logZ, lz, rtol=1e-13)
    assert r.loglik == pytest.approx(lz.sum(), rel=1e-13)


def test_k1_variance_uses_updated_mean():
    """Eq. (3) divides Σ r ‖x − μ_new‖² by N_k: with a far-off input mean the
    result must still be the variance about the sample mean, not about μ_in."""
    rng = np.random.default_rng(2)
    X = rng.normal(size=(100, 3)) + 5.0
    r = O.em_step(X, [1.0], np.zeros((1, 3)), np.ones((1, 3)), O.COV_DIAG, 0.0)
    np.testing.assert_allclose(r.variances[0], X.var(axis=0), rtol=1e-12)


# ----------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("spherical", [False, True])
def test_oracle_matches_brute_force(seed, spherical):
    rng = np.random.default_rng(10 + seed)
    N, K, D = 40 + seed * 7, 3 + seed, 1 + seed
    X, w, mu, var = _rand_problem(rng, N, K, D, spherical)
    cov = O.COV_SPHERICAL if spherical else O.COV_DIAG
    reg = 1e-4
    r = O.em_step(X, w, mu, var, cov, reg)
    bw, bmu, bvar, bll, blz, bR = brute.em_step(X.tolist(), w.tolist(), mu.tolist(),
                                                var.tolist(), spherical, reg)
    np.testing.assert_allclose(r.weights, bw, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r.means, bmu, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.variances, bvar, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.logZ, blz, rtol=1e-13)
    assert r.loglik == pytest.approx(bll, rel=1e-13)
    lz, R = O.e_step(X, w, mu, var, cov)
    np.testing.assert_allclose(R, bR, rtol=1e-11, atol=1e-15)


@pytest.mark.parametrize("seed", [0, 1])
def test_soft_assign_matches_brute_force(seed):
    rng = np.random.default_rng(20 + seed)
    N, K, D = 50, 6, 3
    X, w, mu, var = _rand_problem(rng, N, K, D, spread=1.0)
    for top_m, thr in [(1, 0.0), (2, 1.0 / K), (3, 0.05), (6, 0.0)]:
        ids, resp = O.soft_assign(X, w, mu, var, O.COV_DIAG, top_m, thr)
        bi, br = brute.top_m_assign(X.tolist(), w.tolist(), mu.tolist(), var.tolist(), top_m, thr)
        np.testing.assert_array_equal(ids, np.array(bi))
        np.testing.assert_allclose(resp, br, rtol=1e-12, atol=1e-15)


# ----------------------------------------------------------------- library special cases
@pytest.mark.parametrize("cov", ["diag", "spherical"])
def test_one_step_matches_sklearn(cov):
    """sklearn's GaussianMixture(max_iter=1) from given weights/means/precisions
    runs one E-step and one M-step of the same model (it adds 10·eps to N_k and
    reg_covar to the variances, like our floor)."""
    from sklearn.mixture import GaussianMixture
    import warnings
    rng = np.random.default_rng(3)
    N, K, D = 600, 4, 3
    X, w, mu, var = _rand_problem(rng, N, K, D, spherical=(cov == "spherical"), spread=2.0)
    reg = 1e-5
    gm = GaussianMixture(n_components=K, covariance_type=cov, max_iter=1, reg_covar=reg,
                         weights_init=w, means_init=mu, precisions_init=1.0 / var,
                         init_params="random", random_state=0, tol=0.0)
    # score of the INITIAL parameters: the same object before fitting
    from sklearn.mixture._gaussian_mixture import _compute_precision_cholesky
    ref_init = GaussianMixture(n_components=K, covariance_type=cov)
    ref_init.weights_, ref_init.means_ = w, mu
    ref_init.covariances_ = var
    ref_init.precisions_cholesky_ = _compute_precision_cholesky(var, cov)
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        gm.fit(X)
    c = O.COV_SPHERICAL if cov == "spherical" else O.COV_DIAG
    r = O.em_step(X, w, mu, var, c, reg)
    np.testing.assert_allclose(r.logZ, ref_init.score_samples(X), rtol=1e-11)
    np.testing.assert_allclose(r.weights, gm.weights_, rtol=1e-10)
    np.testing.assert_allclose(r.means, gm.means_, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r.variances, gm.covariances_, rtol=1e-9)


def test_equal_sigma_pi_is_softmax_of_distances():
    """Equal σ and π: r_i = softmax_k(−‖x_i − μ_k‖² / (2σ²)) (textbook softmax)."""
    rng = np.random.default_rng(4)
    N, K, D = 80, 5, 4
    X = rng.normal(size=(N, D))
    mu = rng.normal(size=(K, D))
    s2 = 0.7
    _, R = O.e_step(X, np.full(K, 1.0 / K), mu, np.full((K, D), s2), O.COV_DIAG)
    ref = scipy.special.softmax(-cdist(X, mu, "sqeuclidean") / (2 * s2), axis=1)
    np.testing.assert_allclose(R, ref, rtol=1e-12, atol=1e-15)
    _, Rs = O.e_step(X, np.full(K, 1.0 / K), mu, np.full(K, s2), O.COV_SPHERICAL)
    np.testing.assert_allclose(Rs, ref, rtol=1e-12, atol=1e-15)


def test_small_sigma_limit_is_nearest_mean():
    """σ → 0: responsibilities become the one-hot nearest-mean (Lloyd) assignment."""
    rng = np.random.default_rng(5)
    X = rng.normal(size=(200, 3))
    mu = rng.normal(size=(7, 3))
    _, R = O.e_step(X, np.full(7, 1 / 7), mu, np.full((7, 3), 1e-6), O.COV_DIAG)
    nearest = np.argmin(cdist(X, mu), axis=1)
    np.testing.assert_array_equal(np.argmax(R, axis=1), nearest)
    assert np.all(R.max(axis=1) > 1 - 1e-12)
    ids, _ = O.soft_assign(X, np.full(7, 1 / 7), mu, np.full((7, 3), 1e-6), O.COV_DIAG, 1, 0.0)
    np.testing.assert_array_equal(ids[:, 0], nearest)


def test_two_component_1d_closed_form():
    """1-D, μ = ±1, σ² = 1, π = ½: log N(x|1,1) − log N(x|−1,1) = 2x, so
    r_i1 = 1/(1 + e^{−2x}) (Eq. for r_ik, §2).  One M-step then follows
    Eqs. (1)-(3) written out by hand."""
    x = np.array([-2.0, -0.5, 0.25, 1.0, 3.0])
    r1 = 1.0 / (1.0 + np.exp(-2.0 * x))
    r0 = 1.0 - r1
    res = O.em_step(x[:, None], [0.5, 0.5], [[-1.0], [1.0]], [[1.0], [1.0]], O.COV_DIAG, 0.0)
    n0, n1 = r0.sum(), r1.sum()
    m0, m1 = (r0 * x).sum() / n0, (r1 * x).sum() / n1
    v0, v1 = (r0 * (x - m0) ** 2).sum() / n0, (r1 * (x - m1) ** 2).sum() / n1
    np.testing.assert_allclose(res.weights, [n0 / 5, n1 / 5], rtol=1e-14)
    np.testing.assert_allclose(res.means[:, 0], [m0, m1], rtol=1e-14)
    np.testing.assert_allclose(res.variances[:, 0], [v0, v1], rtol=1e-13)
    lz = np.log(0.5 * np.exp(-0.5 * (x + 1) ** 2) + 0.5 * np.exp(-0.5 * (x - 1) ** 2)) \
        - 0.5 * math.log(2 * math.pi)
    np.testing.assert_allclose(res.logZ, lz, rtol=1e-14)


# ----------------------------------------------------------------- invariants
def test_responsibilities_are_a_distribution():
    rng = np.random.default_rng(6)
    X, w, mu, var = _rand_problem(rng, 300, 9, 6)
    _, R = O.e_step(X, w, mu, var, O.COV_DIAG)
    assert np.all(R >= 0) and np.all(R <= 1)
    np.testing.assert_allclose(R.sum(axis=1), 1.0, rtol=1e-14)


def test_fit_tolerance_rule_from_the_k1_fixed_point():
    """§2's stopping rule (a small change of the log-likelihood between successive
    iterations), read as |L_t - L_(t-1)| / N < tol.  With K = 1 the first step lands on
    the maximum-likelihood parameters (closed form: sample mean, population variance)
    and every later step returns them unchanged, so L_1 = L_2 exactly and the change
    seen after iteration 3 is 0, while the change after iteration 2 is
    d1 = |L(MLE) - L(Θ_0)| / N > 0.  Hence: tol = 0 runs every iteration; any tol in
    (0, d1] stops after 3 (d1 < tol is false at d1 itself: strict); tol above d1 stops
    after 2.  A rule without the division by N, or with <= instead of <, fails."""
    rng = np.random.default_rng(31)
    N, D = 400, 3
    X = rng.normal(loc=[1.0, -1.0, 2.0], scale=[0.5, 1.5, 1.0], size=(N, D))
    mu0, var0 = np.zeros((1, D)), np.full((1, D), 3.0)
    _, mu_a, var_a, lls, it = O.fit(X, [1.0], mu0, var0, max_iters=6, tol=0.0)
    assert it == 6 and len(lls) == 6
    np.testing.assert_allclose(mu_a[0], X.mean(axis=0), rtol=1e-13)
    np.testing.assert_allclose(var_a[0], X.var(axis=0) + 1e-6, rtol=1e-12)
    assert lls[1] == lls[2]            # the fixed point: identical parameters, identical L
    d1 = abs(lls[1] - lls[0]) / N
    assert d1 > 0
    for tol, want in ((1e-300, 3), (0.5 * d1, 3), (d1, 3), (2.0 * d1, 2)):
        *_, lls_t, it_t = O.fit(X, [1.0], mu0, var0, max_iters=6, tol=tol)
        assert it_t == want, (tol, d1, it_t)
        assert lls_t == lls[:want]


@pytest.mark.parametrize("cov", [O.COV_DIAG, O.COV_SPHERICAL])
def test_loglik_monotone(cov):
    """EM never decreases the likelihood (Dempster et al. 1977, cited in §2)."""
    rng = np.random.default_rng(7)
    K, D, N = 5, 3, 1500
    centers = rng.normal(size=(K, D)) * 2.5
    X = centers[rng.integers(0, K, N)] + rng.normal(size=(N, D))
    mu = X[rng.choice(N, K, replace=False)]
    var = np.full(K, 2.0) if cov == O.COV_SPHERICAL else np.full((K, D), 2.0)
    _, _, _, lls, _ = O.fit(X, np.full(K, 1 / K), mu, var, cov, reg_covar=0.0, max_iters=40)
    assert np.all(np.isfinite(lls))
    d = np.diff(lls)
    assert np.all(d >= -1e-7 * np.abs(np.array(lls[1:])))


def test_component_permutation_equivariance():
    rng = np.random.default_rng(8)
    X, w, mu, var = _rand_problem(rng, 150, 5, 3)
    p = rng.permutation(5)
    a = O.em_step(X, w, mu, var)
    b = O.em_step(X, w[p], mu[p], var[p])
    np.testing.assert_allclose(b.weights, a.weights[p], rtol=1e-13)
    np.testing.assert_allclose(b.means, a.means[p], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b.variances, a.variances[p], rtol=1e-12)
    assert b.loglik == pytest.approx(a.loglik, rel=1e-14)


def test_row_permutation_invariance():
    rng = np.random.default_rng(9)
    X, w, mu, var = _rand_problem(rng, 150, 5, 3)
    p = rng.permutation(150)
    a = O.em_step(X, w, mu, var)
    b = O.em_step(X[p], w, mu, var)
    np.testing.assert_allclose(b.means, a.means, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b.variances, a.variances, rtol=1e-12)
    np.testing.assert_allclose(b.logZ, a.logZ[p], rtol=1e-14)


def test_row_chunking_does_not_change_results(monkeypatch):
    rng = np.random.default_rng(11)
    X, w, mu, var = _rand_problem(rng, 500, 7, 3)
    a = O.em_step(X, w, mu, var)
    monkeypatch.setattr(O, "_CHUNK_BYTES", 8 * 7 * 3 * 37)  # 37-row chunks
    b = O.em_step(X, w, mu, var)
    np.testing.assert_allclose(b.means, a.means, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(b.variances, a.variances, rtol=1e-13)
    np.testing.assert_allclose(b.logZ, a.logZ, rtol=1e-15)


# ----------------------------------------------------------------- empty components
def test_dead_component_is_kept_and_zero_weighted():
    rng = np.random.default_rng(12)
    X = rng.normal(size=(100, 2))
    mu = np.array([[0.0, 0.0], [1.0, 1.0], [1e4, 1e4]])  # third is unreachable
    var = np.ones((3, 2))
    r = O.em_step(X, np.full(3, 1 / 3), mu, var, O.COV_DIAG, 1e-6)
    assert r.empty.tolist() == [False, False, True]
    assert r.weights[2] == 0.0
    np.testing.assert_array_equal(r.means[2], mu[2])
    np.testing.assert_array_equal(r.variances[2], var[2])
    assert r.weights[:2].sum() == pytest.approx(1.0, abs=1e-15)
    # the next step excludes it entirely (log π = −inf)
    r2 = O.em_step(X, r.weights, r.means, r.variances)
    assert np.all(np.isfinite(r2.logZ))
    _, R = O.e_step(X, r.weights, r.means, r.variances)
    assert np.all(R[:, 2] == 0.0)


def test_all_empty_is_an_error():
    X = np.zeros((3, 1))
    with pytest.raises(FloatingPointError):
        O.em_step(X, [0.0, 0.0], [[0.0], [1.0]], [[1.0], [1.0]])


# ----------------------------------------------------------------- soft assign semantics
def test_soft_assign_threshold_and_ties():
    """Ranks 2..m need r > τ strictly; rank 1 is always kept; equal scores go
    to the lower component index (§4.3)."""
    X = np.array([[0.0], [0.5], [10.0]])
    mu = np.array([[0.0], [0.0], [1.0]])          # components 0 and 1 identical
    var = np.ones((3, 1))
    w = np.full(3, 1 / 3)
    ids, resp = O.soft_assign(X, w, mu, var, O.COV_DIAG, top_m=3, r_threshold=0.0)
    assert ids[0, 0] == 0 and ids[0, 1] == 1     # tie broken by index
    assert resp[0, 0] == resp[0, 1]
    # the point at 10 is far closer to component 2: ranks 2, 3 are tiny but > 0
    assert ids[2, 0] == 2
    ids, resp = O.soft_assign(X, w, mu, var, O.COV_DIAG, top_m=3, r_threshold=0.34)
    assert ids[2].tolist() == [2, -1, -1] and resp[2, 1] == 0.0
    # top-1 is the argmax of the dense responsibilities
    _, R = O.e_step(X, w, mu, var)
    ids1, resp1 = O.soft_assign(X, w, mu, var, O.COV_DIAG, 1, 0.99)
    np.testing.assert_array_equal(ids1[:, 0], np.argmax(R, axis=1))
    np.testing.assert_allclose(resp1[:, 0], R.max(axis=1), rtol=1e-15)


# ----------------------------------------------------------------- recovery
def test_recovers_well_separated_mixture():
    """A seeded mixture with means far apart (≥ 10σ): EM from one data point per
    cluster recovers means within sampling error and weights within ~3/√N."""
    rng = np.random.default_rng(13)
    K, D, N = 4, 3, 4000
    true_mu = np.array([[0, 0, 0], [12, 0, 0], [0, 12, 0], [0, 0, 12]], dtype=float)
    true_w = np.array([0.1, 0.2, 0.3, 0.4])
    true_s = np.array([0.5, 1.0, 1.5, 0.8])
    lab = rng.choice(K, N, p=true_w)
    X = true_mu[lab] + true_s[lab, None] * rng.normal(size=(N, D))
    init = np.array([X[np.nonzero(lab == k)[0][0]] for k in range(K)])
    w, mu, var, lls, _ = O.fit(X, np.full(K, 1 / K), init, np.ones((K, D)), O.COV_DIAG,
                               1e-6, max_iters=30)
    for k in range(K):
        nk = (lab == k).sum()
        assert np.all(np.abs(mu[k] - true_mu[k]) < 4 * true_s[k] / math.sqrt(nk))
        assert abs(w[k] - true_w[k]) < 3 * math.sqrt(true_w[k] / N) + 1e-3
        np.testing.assert_allclose(np.sqrt(var[k]), true_s[k], rtol=0.1)


# ------------------------------------------------------------------ sharded statistics
@pytest.mark.parametrize("spherical", [False, True])
def test_shard_statistics_match_brute_force(spherical):
    """The exchanged statistics (N_k, Σ r (x − μ), Σ r (x − μ)² about the input
    mean, Σ log Z) against the pure-Python statement on a tiny input."""
    rng = np.random.default_rng(11)
    N, K, D = 23, 3, 2
    X = rng.normal(size=(N, D)) * 2.0
    w = np.array([0.5, 0.3, 0.2])
    mu = rng.normal(size=(K, D))
    var = rng.uniform(0.5, 2.0, size=K) if spherical else rng.uniform(0.5, 2.0, size=(K, D))
    cov = O.COV_SPHERICAL if spherical else O.COV_DIAG
    got = O.shard_statistics(X, w, mu, var, cov)
    ref = brute.shard_statistics(X.tolist(), w.tolist(), mu.tolist(), var.tolist(), spherical)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_shard_statistics_are_additive_over_row_partitions():
    """Every entry is a sum over rows: three uneven shards add up to the whole."""
    rng = np.random.default_rng(12)
    X = rng.normal(size=(700, 6))
    K = 5
    w = rng.dirichlet(np.ones(K))
    mu = X[rng.choice(700, K, replace=False)]
    var = rng.uniform(0.5, 2.0, size=(K, 6))
    parts = [X[:1], X[1:333], X[333:]]
    tot = sum(O.shard_statistics(p, w, mu, var) for p in parts)
    np.testing.assert_allclose(tot, O.shard_statistics(X, w, mu, var), rtol=1e-12, atol=1e-9)


@pytest.mark.parametrize("cov", [O.COV_DIAG, O.COV_SPHERICAL])
def test_m_step_from_statistics_equals_em_step(cov):
    """Eq. (3) about the updated mean follows from the sums about the input mean:
    the M-step on summed shard statistics equals the one-pass em_step."""
    rng = np.random.default_rng(13)
    X = np.concatenate([rng.normal(-3, 1, size=(300, 4)), rng.normal(2, 0.5, size=(200, 4))])
    K = 3
    w = np.full(K, 1 / K)
    mu = X[[0, 1, 350]]
    var = np.ones(K) if cov == O.COV_SPHERICAL else np.ones((K, 4))
    st = O.shard_statistics(X[:137], w, mu, var, cov) + O.shard_statistics(X[137:], w, mu, var, cov)
    a = O.m_step_from_statistics(st, w, mu, var, cov)
    b = O.em_step(X, w, mu, var, cov)
    np.testing.assert_allclose(a.means, b.means, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(a.variances, b.variances, rtol=1e-10)
    np.testing.assert_allclose(a.weights, b.weights, rtol=1e-12)
    assert abs(a.loglik - b.loglik) <= 1e-12 * abs(b.loglik)


def test_m_step_from_statistics_keeps_empty_components():
    """A component with N_k below the empty threshold keeps μ, σ² and gets π = 0."""
    K, D = 2, 3
    st = np.zeros(K * (1 + 2 * D) + 1)
    st[0] = 10.0
    st[1:1 + D] = [1.0, 2.0, 3.0]
    st[1 + D:1 + 2 * D] = [10.0, 10.0, 10.0]
    st[-1] = -5.0
    mu = np.array([[0.0, 0.0, 0.0], [7.0, 8.0, 9.0]])
    var = np.array([[1.0, 1.0, 1.0], [4.0, 5.0, 6.0]])
    r = O.m_step_from_statistics(st, np.array([0.5, 0.5]), mu, var, reg_covar=0.0)
    np.testing.assert_allclose(r.means[0], [0.1, 0.2, 0.3])
    np.testing.assert_allclose(r.variances[0], [1 - 0.01, 1 - 0.04, 1 - 0.09])
    np.testing.assert_array_equal(r.means[1], mu[1])
    np.testing.assert_array_equal(r.variances[1], var[1])
    np.testing.assert_array_equal(r.weights, [1.0, 0.0])
    assert r.loglik == -5.0


# ------------------------------------------------------------------ Fisher vectors
@pytest.mark.parametrize("spherical", [False, True])
def test_fisher_vector_matches_brute_force(spherical):
    rng = np.random.default_rng(31)
    N, K, D = 17, 3, 2
    X = rng.normal(size=(N, D)) * 2
    w = np.array([0.2, 0.5, 0.3])
    mu = rng.normal(size=(K, D))
    var = rng.uniform(0.5, 2.0, size=K) if spherical else rng.uniform(0.5, 2.0, size=(K, D))
    cov = O.COV_SPHERICAL if spherical else O.COV_DIAG
    got = O.fisher_vector(X, w, mu, var, cov)
    ref = brute.fisher_vector(X.tolist(), w.tolist(), mu.tolist(), var.tolist(), spherical)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_fisher_vector_single_gaussian_closed_form():
    """K = 1 at the sample mean: G_mu = 0; G_sigma_d = (s_d^2 / sigma_d^2 - 1) / sqrt(2),
    with s_d^2 the (1/N) sample variance."""
    rng = np.random.default_rng(32)
    X = rng.normal(size=(400, 3)) * [1.0, 2.0, 0.5] + [3.0, -1.0, 0.0]
    mu = X.mean(0, keepdims=True)
    var = np.array([[1.5, 3.0, 0.2]])
    fv = O.fisher_vector(X, np.array([1.0]), mu, var)
    np.testing.assert_allclose(fv[:3], 0.0, atol=1e-12)
    np.testing.assert_allclose(fv[3:], (X.var(0) / var[0] - 1.0) / np.sqrt(2.0), rtol=1e-12)


def test_fisher_vector_normalisation():
    rng = np.random.default_rng(33)
    X = rng.normal(size=(50, 2))
    w, mu, var = np.array([0.5, 0.5]), np.array([[-1.0, 0.0], [1.0, 0.0]]), np.ones((2, 2))
    raw = O.fisher_vector(X, w, mu, var)
    fv = O.fisher_vector(X, w, mu, var, normalize=True)
    assert abs(np.linalg.norm(fv) - 1.0) < 1e-12
    np.testing.assert_allclose(fv * np.linalg.norm(np.sqrt(np.abs(raw))),
                               np.sign(raw) * np.sqrt(np.abs(raw)), rtol=1e-12, atol=1e-15)
