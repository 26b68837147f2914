"""Golden fixtures (tests/golden/*.json, written by tests/golden/make_golden.py from the
oracle alone): the oracle must keep reproducing them (CPU), and the CUDA path must
match them (GPU, marked)."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import gmm_oracle as O
from oracle import kmeans_oracle as KM

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("case,cov", [("diag", O.COV_DIAG), ("spherical", O.COV_SPHERICAL)])
def test_oracle_reproduces_the_em_fixture(case, cov):
    g = _load("tiny_em.json")
    c = g[case]
    r = O.em_step(np.array(g["X"]), np.array(g["weights_in"]), np.array(g["means_in"]),
                  np.array(c["var_in"]), cov, g["reg_covar"])
    np.testing.assert_allclose(r.means, c["means"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r.variances, c["variances"], rtol=1e-13)
    np.testing.assert_allclose(r.weights, c["weights"], rtol=1e-13)
    assert abs(r.loglik - c["loglik"]) <= 1e-12 * abs(c["loglik"])
    assert abs(sum(c["weights"]) - 1.0) < 1e-12


def test_oracle_reproduces_the_kmeans_fixture():
    g = _load("tiny_kmeans.json")
    X = np.array(g["X"], dtype=np.float32)
    C, a, counts, inertia = KM.lloyd_step(X, np.array(g["C0"], dtype=np.float32))
    assert a.tolist() == g["assign"] and counts.tolist() == g["counts"]
    np.testing.assert_allclose(C, g["centroids"], rtol=1e-15)
    idx, _ = KM.kmeanspp(X, len(g["seed_u"]) + 1, g["seed_first"], g["seed_u"])
    assert idx.tolist() == g["seed_idx"]


@pytest.mark.gpu
@pytest.mark.parametrize("case,prec", [("diag", "fp32"), ("diag", "auto"), ("spherical", "fp32"),
                                       ("spherical", "fp16x3")])
def test_cuda_em_step_matches_the_fixture(case, prec):
    import ivf_quantizer_b200 as q
    g = _load("tiny_em.json")
    c = g[case]
    cov = q.COV_DIAG if case == "diag" else q.COV_SPHERICAL
    h = q.GMM(3, 2, cov, g["reg_covar"])
    h.set_precision({"fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO}[prec])
    X = torch.tensor(g["X"], dtype=torch.float32, device="cuda")
    w, mu, var = h.new_params(g["weights_in"], g["means_in"], c["var_in"])
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(X.shape[0], dtype=torch.float32, device="cuda")
    h.step(X, w, mu, var, loglik=ll, logz=lz)
    torch.cuda.synchronize()
    assert h.status() == 0
    np.testing.assert_allclose(lz.cpu().numpy(), c["logZ"], rtol=1e-4)
    np.testing.assert_allclose(mu.cpu().numpy(), c["means"], rtol=1e-3, atol=1e-3)
    np.testing.assert_allclose(var.cpu().numpy(), c["variances"], rtol=1e-3)
    np.testing.assert_allclose(w.cpu().numpy(), c["weights"], rtol=1e-3)
    assert abs(ll.item() - c["loglik"]) <= 1e-4 * abs(c["loglik"])
    if prec == "fp32":
        w0, mu0, var0 = h.new_params(g["weights_in"], g["means_in"], c["var_in"])
        ids, resp = h.soft_assign(X, w0, mu0, var0, top_m=g["top_m"], r_threshold=g["r_threshold"])
        torch.cuda.synchronize()
        assert ids.cpu().tolist() == c["soft_ids"]
        np.testing.assert_allclose(resp.cpu().numpy(), c["soft_resp"], rtol=1e-4, atol=1e-6)
    h.close()


@pytest.mark.gpu
def test_cuda_kmeans_matches_the_fixture():
    import ivf_quantizer_b200 as q
    g = _load("tiny_kmeans.json")
    X = torch.tensor(g["X"], dtype=torch.float32, device="cuda")
    h = q.GMM(len(g["C0"]), 2)
    C = torch.tensor(g["C0"], dtype=torch.float32, device="cuda")
    a = torch.empty(X.shape[0], dtype=torch.int32, device="cuda")
    cnt = torch.empty(len(g["C0"]), dtype=torch.int64, device="cuda")
    h.kmeans_step(X, C, assign=a, counts=cnt)
    torch.cuda.synchronize()
    assert a.cpu().tolist() == g["assign"] and cnt.cpu().tolist() == g["counts"]
    np.testing.assert_allclose(C.cpu().numpy(), g["centroids"], rtol=2e-7, atol=1e-7)
    h.close()
    h = q.GMM(len(g["seed_u"]) + 1, 2)
    _, idx = h.kmeans_seed(X, g["seed_first"], g["seed_u"])
    torch.cuda.synchronize()
    assert idx.cpu().tolist() == g["seed_idx"]
    h.close()
