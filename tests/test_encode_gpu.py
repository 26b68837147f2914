"""Per-point scoring (fgmm_score_samples, KDE use) and Fisher-vector encoding
(fgmm_fisher_vector) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import gmm_oracle as O

pytestmark = pytest.mark.gpu


def _g(K, D, prec, cov=0):
    import ivf_quantizer_b200 as q
    g = q.GMM(K, D, cov)
    g.set_precision({"fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO}[prec])
    return g


@pytest.mark.parametrize("prec", ["fp32", "fp16x3", "auto"])
@pytest.mark.parametrize("gen,N,K", [("c1", 7000, 16), ("table1", 3000, 64)])
def test_score_samples_matches_oracle(prec, gen, N, K):
    X = synth.generate(gen, N, seed=21)
    w, mu, var = synth.init_params(X, K, seed=21)
    g = _g(K, X.shape[1], prec)
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = g.score_samples(X.cuda(), wd, md, vd, loglik=ll)
    torch.cuda.synchronize()
    assert g.status() == 0
    # parameters untouched
    assert torch.equal(wd.cpu(), w.float()) and torch.equal(md.cpu(), mu.float())
    ref = O.logsumexp_rows(O.log_joint(X.double().numpy(), w.double().numpy(),
                                       mu.double().numpy(), var.double().numpy()))
    assert np.max(np.abs(lz.cpu().numpy() - ref) / np.abs(ref)) <= 1e-4
    assert abs(ll.item() - ref.sum()) <= 1e-4 * abs(ref.sum())
    g.close()


def test_kde_with_equal_weights_and_shared_bandwidth():
    import ivf_quantizer_b200 as q
    rng = np.random.default_rng(3)
    sample = rng.normal(size=(200, 4)).astype(np.float32)
    Y = rng.normal(size=(1000, 4)).astype(np.float32)
    h2 = 0.3
    g = q.GMM(200, 4, q.COV_SPHERICAL)
    g.set_precision(q.PREC_FP32)
    w, mu, var = g.new_params(np.full(200, 1 / 200), sample, np.full(200, h2))
    lz = g.score_samples(torch.from_numpy(Y).cuda(), w, mu, var).cpu().numpy()
    # direct KDE: log mean_j N(y | s_j, h2 I)
    d2 = ((Y[:, None, :].astype(np.float64) - sample[None].astype(np.float64)) ** 2).sum(-1)
    logk = -0.5 * d2 / h2 - 2.0 * np.log(2 * np.pi * h2)
    m = logk.max(1)
    ref = m + np.log(np.exp(logk - m[:, None]).mean(1))
    assert np.max(np.abs(lz - ref) / np.abs(ref)) <= 1e-4
    g.close()


@pytest.mark.parametrize("prec,cov", [("fp32", 0), ("fp32", 1), ("auto", 0)])
@pytest.mark.parametrize("normalize", [False, True])
def test_fisher_vector_matches_oracle(prec, cov, normalize):
    X = synth.generate("c1", 6000, seed=22)
    w, mu, var = synth.init_params(X, 16, seed=22)
    if cov == 1:
        var = var.mean(1)
    g = _g(16, 16, prec, cov)
    wd, md, vd = g.new_params(w, mu, var)
    fv = g.fisher_vector(X.cuda(), wd, md, vd, normalize=normalize).cpu().numpy()
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = O.fisher_vector(X.double().numpy(), w.double().numpy(), mu.double().numpy(),
                          var.double().numpy(), cov, normalize=normalize)
    scale = np.max(np.abs(ref))
    # G_sigma is a difference of comparable sums: judged on the vector's scale
    tol = 1e-4 if prec == "fp32" else 2e-3
    assert np.max(np.abs(fv - ref)) <= tol * scale, np.max(np.abs(fv - ref)) / scale
    g.close()
