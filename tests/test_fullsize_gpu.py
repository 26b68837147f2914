"""Parity at the full benchmark size (N = 100,000,000, D = 128, K = 1024, diagonal,
fp32 X resident in HBM), in the launch configuration bench.py times.

The oracle cannot run a whole step at this size, so the test checks per-point
log-likelihoods on sampled rows one by one against the oracle, and properties
that hold at any size: the step's log-likelihood equals the fp64 sum of the
per-point values, the weights form a distribution, every parameter is finite
and positive where it must be, and device memory beyond X does not grow.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gmm_oracle as O

pytestmark = pytest.mark.gpu

N, D, K = 100_000_000, 128, 1024


@pytest.fixture(scope="module")
def big_x():
    if torch.cuda.get_device_properties(0).total_memory < 120e9:
        pytest.skip("needs a 180 GB device")
    X = torch.empty(N, D, device="cuda", dtype=torch.float32)
    synth.generate("table1", N, seed=0, device="cuda", out=X)
    yield X
    del X
    torch.cuda.empty_cache()


@pytest.mark.parametrize("prec", ["auto", "fp16x3"])
def test_full_size_step(big_x, prec):
    import ivf_quantizer_b200 as q
    X = big_x
    w, mu, var = synth.init_params(X, K, seed=0)
    g = q.GMM(K, D)
    g.set_precision({"auto": q.PREC_AUTO, "fp16x3": q.PREC_FP16X3}[prec])
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(N, dtype=torch.float32, device="cuda")
    # a first step on a small slice loads every kernel (lazy module loading allocates
    # then); the full-size step must not change device memory after that
    w2, m2, v2 = wd.clone(), md.clone(), vd.clone()
    g.step(X[:8192], w2, m2, v2)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    g.step(X, wd, md, vd, loglik=ll, logz=lz)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert g.status() == 0
    # sampled per-point log-likelihoods, one by one against the oracle
    gen = torch.Generator().manual_seed(123)
    rows = torch.cat([torch.randint(0, N, (3000,), generator=gen),
                      torch.tensor([0, 1, (1 << 20) - 1, 1 << 20, N - 129, N - 1])])
    xs = X[rows.cuda()].double().cpu().numpy()
    L = O.log_joint(xs, w.double().numpy(), mu.double().numpy(), var.double().numpy())
    ref = O.logsumexp_rows(L)
    got = lz[rows.cuda()].double().cpu().numpy()
    rel = np.abs(got - ref) / np.abs(ref)
    assert rel.max() <= 1e-4, rel.max()
    # the step's log-likelihood is the sum of the per-point values
    total = float(lz.double().sum().item())
    assert abs(total - ll.item()) <= 1e-9 * abs(total)
    wn = wd.double().cpu().numpy()
    assert abs(wn.sum() - 1.0) < 1e-5 and np.all(wn >= 0)
    assert torch.isfinite(md).all() and torch.isfinite(vd).all() and bool((vd > 0).all())
    g.close()
