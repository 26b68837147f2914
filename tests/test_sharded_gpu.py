"""Sharded EM on one GPU: fgmm_em_partial on row shards, fgmm_stats_sum, then
fgmm_em_finish, against the fp64 oracle on the union of the shards (the multi-rank
orchestration itself is covered on CPU in test_dist_cpu.py)."""
import numpy as np
import pytest
import torch

import synth
from oracle import gmm_oracle as O
from tests._cmp import compare_step

pytestmark = pytest.mark.gpu


def _engine(K, D, prec, cov=0):
    import ivf_quantizer_b200 as q
    g = q.GMM(K, D, cov)
    g.set_precision({"fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO}[prec])
    return g


@pytest.mark.parametrize("prec", ["fp32", "fp16x3", "auto"])
@pytest.mark.parametrize("cuts", [[0, 4000, 10000], [0, 1, 5000, 10000]])
def test_shards_summed_equal_the_union(prec, cuts):
    import ivf_quantizer_b200 as q
    X = synth.generate("c1", 10_000, seed=4)
    w, mu, var = synth.init_params(X, 16, seed=4)
    g = _engine(16, X.shape[1], prec)
    Xd = X.cuda()
    wd, md, vd = g.new_params(w, mu, var)
    parts = torch.stack([g.partial(Xd[a:b], wd, md, vd) for a, b in zip(cuts[:-1], cuts[1:])])
    tot = q.stats_sum(parts.contiguous())
    # the sum is taken in part order
    seq = parts[0].clone()
    for p in parts[1:]:
        seq += p
    assert torch.equal(tot, seq)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    g.finish(tot, wd, md, vd, loglik=ll)
    torch.cuda.synchronize()
    assert g.status() == 0
    ref = O.em_step(X.double().numpy(), w.double().numpy(), mu.double().numpy(),
                    var.double().numpy())
    print(compare_step((wd.cpu().numpy(), md.cpu().numpy(), vd.cpu().numpy()), ref,
                       X.numpy(), loglik_gpu=float(ll.item())))
    # the statistics vector itself against the oracle's: N_k and the log-likelihood
    st = O.shard_statistics(X.double().numpy(), w.double().numpy(), mu.double().numpy(),
                            var.double().numpy())
    got = tot.cpu().numpy()
    D = X.shape[1]
    nk, nk_ref = got[:-1].reshape(16, 1 + 2 * D)[:, 0], st[:-1].reshape(16, 1 + 2 * D)[:, 0]
    big = nk_ref >= 1.0
    assert np.max(np.abs(nk[big] - nk_ref[big]) / nk_ref[big]) <= 1e-3
    assert abs(got[-1] - st[-1]) <= 1e-4 * abs(st[-1])
    g.close()


@pytest.mark.parametrize("prec", ["fp32", "auto"])
def test_step_is_partial_then_finish(prec):
    """fgmm_em_step and fgmm_em_partial + fgmm_em_finish give bit-identical parameters
    (two handles in the same state: under AUTO a handle remembers the previous step's
    N_k, which steers the next step's per-component path)."""
    X = synth.generate("table1", 5000, seed=5).cuda()
    w, mu, var = synth.init_params(X.cpu(), 64, seed=5)
    g, h = _engine(64, 128, prec), _engine(64, 128, prec)
    a = g.new_params(w, mu, var)
    b = h.new_params(w, mu, var)
    la = torch.zeros(1, dtype=torch.float64, device="cuda")
    lb = torch.zeros(1, dtype=torch.float64, device="cuda")
    for _ in range(2):
        g.step(X, *a, loglik=la)
        st = h.partial(X, *b)
        h.finish(st, *b, loglik=lb)
        torch.cuda.synchronize()
        assert g.status() == 0 and h.status() == 0
        for ta, tb in zip(a, b):
            assert torch.equal(ta, tb)
        assert torch.equal(la, lb)
        assert float(st[-1].item()) == float(la.item())
    g.close()
    h.close()


def test_finish_with_non_finite_loglik_keeps_parameters():
    import ivf_quantizer_b200 as q
    X = synth.generate("c1", 2000, seed=6).cuda()
    w, mu, var = synth.init_params(X.cpu(), 16, seed=6)
    g = _engine(16, X.shape[1], "fp32")
    wd, md, vd = g.new_params(w, mu, var)
    st = g.partial(X, wd, md, vd)
    st[-1] = float("nan")
    w0, m0, v0 = wd.clone(), md.clone(), vd.clone()
    g.finish(st, wd, md, vd)
    assert g.status() == q._lib.ERR_NUMERIC
    assert torch.equal(wd, w0) and torch.equal(md, m0) and torch.equal(vd, v0)
    g.close()
