"""Soft assignment (§4.2-4.3) with the tensor-core filter.

With the split-product modes and 2 to 32 component blocks, fgmm_soft_assign runs the
log-sum-exp sweep on the tensor cores with every component to mark, per point, the
128-component blocks whose log-densities come within a cut of log Z (widened by the
expanded form's error bound), regroups the points by those marks, and evaluates only
the marked blocks exactly on CUDA cores, with the dense kernel's arithmetic.  The ids
must therefore equal the dense CUDA-core path's (FGMM_PREC_FP32) exactly, the
responsibilities to fp32 rounding (log Z sums in another order), and both must match
the oracle where the decision is not within 1e-3.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gmm_oracle as O
from tests._cmp import ids_match_where_decisive

pytestmark = pytest.mark.gpu


def _assign(X, w, mu, var, prec, top_m, thr, profile=False):
    import ivf_quantizer_b200 as q
    K, D = mu.shape
    g = q.GMM(K, D, precision=prec)
    wd, md, vd = g.new_params(w, mu, var)
    if profile:
        g.profile(True)
        g.profile_read(reset=True)
    ids, resp = g.soft_assign(X, wd, md, vd, top_m=top_m, r_threshold=thr)
    torch.cuda.synchronize()
    kern = g.profile_read(reset=True)["kernels"] if profile else {}
    assert g.status() == 0
    g.close()
    return ids.cpu().numpy(), resp.cpu().numpy(), kern


def _check(gen, N, K, seed, top_m, thr, dtype=torch.float32, var_scale=1.0, steps=2):
    import ivf_quantizer_b200 as q
    X = synth.generate(gen, N, seed=seed).to(dtype)
    w, mu, var = synth.init_params(X.float(), K, seed=seed)
    # a few EM steps so that the components have found their clusters
    g = q.GMM(K, X.shape[1])
    wd, md, vd = g.new_params(w, mu, var * var_scale)
    Xd = X.cuda()
    for _ in range(steps):
        g.step(Xd, wd, md, vd)
    g.check_status()
    w2, m2, v2 = wd.cpu(), md.cpu(), vd.cpu()
    g.close()
    ids_t, resp_t, kern = _assign(Xd, w2, m2, v2, q.PREC_AUTO, top_m, thr, profile=True)
    assert kern.get("tc_lse", {}).get("launches", 0) >= 1, kern   # the tensor-core filter ran
    ids_d, resp_d, _ = _assign(Xd, w2, m2, v2, q.PREC_FP32, top_m, thr)
    np.testing.assert_array_equal(ids_t, ids_d)
    np.testing.assert_allclose(resp_t, resp_d, rtol=2e-5, atol=1e-30)
    Xn = X.float().double().numpy()
    wn, mn, vn = (t.double().numpy() for t in (w2, m2, v2))
    rid, rresp = O.soft_assign(Xn, wn, mn, vn, 0, top_m, thr)
    _, R = O.e_step(Xn, wn, mn, vn)
    decisive, bad = ids_match_where_decisive(ids_t, rid, rresp, R, thr)
    # (with tau = 0 every rank whose r is near 0 is undecided, so count, not fraction)
    assert decisive.sum() >= 50 and len(bad) == 0, (decisive.mean(), bad[:10])
    return ids_t


@pytest.mark.parametrize("gen,N,K,seed,top_m,thr", [
    ("table1", 6000 + 37, 256, 40, 2, 1.0 / 256),     # two blocks, tau = 1/K
    ("table1", 5000, 1024, 41, 2, 0.1),               # eight blocks, the IVF rule
    ("ivf", 8000 + 5, 1024, 42, 2, 0.1),              # anisotropic clusters, Zipf sizes
    ("table1", 3000, 384, 43, 4, 0.0),                # tau = 0: every positive r kept
])
def test_tensor_filtered_assignment_matches_dense_and_oracle(gen, N, K, seed, top_m, thr):
    ids = _check(gen, N, K, seed, top_m, thr)
    if thr == 0.0:
        assert (ids >= 0).sum(1).mean() > 1.5   # the wide cut kept the far ranks


def test_tensor_filtered_assignment_bf16_input():
    _check("table1", 4000, 512, 44, 2, 0.05, dtype=torch.bfloat16)


def test_tensor_filtered_assignment_with_collapsed_components():
    """Components collapsed onto single points (variance 1e-6): their expanded-form
    logit-error bound is far above the filter's limit, so they leave the tensor-core pass
    and are evaluated exactly for every point; the others keep a narrow cut."""
    import ivf_quantizer_b200 as q
    N, K = 5000, 512
    X = synth.generate("table1", N, seed=46)
    w, mu, var = synth.init_params(X, K, seed=46)
    var = var.clone()
    var[[3, 100, 257, 400]] = 1e-6
    Xd = X.cuda()
    ids_t, resp_t, kern = _assign(Xd, w, mu, var, q.PREC_AUTO, 2, 0.05, profile=True)
    assert kern["tc_lse"]["launches"] == 1
    ids_d, resp_d, _ = _assign(Xd, w, mu, var, q.PREC_FP32, 2, 0.05)
    np.testing.assert_array_equal(ids_t, ids_d)
    np.testing.assert_allclose(resp_t, resp_d, rtol=2e-5, atol=1e-30)
    # the collapsed components own the points they sit on
    for k in (3, 100, 257, 400):
        assert np.any(ids_t[:, 0] == k)


def test_tensor_filtered_assignment_across_chunks():
    """N past one 2^20-point chunk with a ragged tail, broad components (several blocks
    per point): per-chunk ordering and write-back to the original indices."""
    import ivf_quantizer_b200 as q
    N, K = (1 << 20) + 1001, 256
    X = synth.generate("table1", N, seed=45).cuda()
    w, mu, var = synth.init_params(X.cpu(), K, seed=45)
    var = var * 4.0
    ids_t, resp_t, kern = _assign(X, w, mu, var, q.PREC_AUTO, 2, 0.05, profile=True)
    assert kern["tc_lse"]["launches"] == 2
    ids_d, resp_d, _ = _assign(X, w, mu, var, q.PREC_FP32, 2, 0.05)
    np.testing.assert_array_equal(ids_t, ids_d)
    np.testing.assert_allclose(resp_t, resp_d, rtol=2e-5, atol=1e-30)
