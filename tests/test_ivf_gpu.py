"""GPU IVF build and search against the oracle: lists, result ids and DCO bit-exact
(both sides rank by the same fp32 operation sequence), distances bit-equal."""
import numpy as np
import pytest
import torch

import synth
from oracle import ivf_oracle as IVF

pytestmark = pytest.mark.gpu


def _index(N, K, D, seed, top_m=2, thr=0.1):
    import ivf_quantizer_b200 as q
    from ivf_quantizer_b200.ivf import IVFIndex
    X = synth.generate("c1", N, seed=seed) if D == 16 else synth.generate("table1", N, seed=seed)
    w, mu, var = synth.init_params(X, K, seed=seed)
    g = q.GMM(K, X.shape[1])
    Xd = X.cuda()
    wd, md, vd = g.new_params(w, mu, var)
    for _ in range(3):
        g.step(Xd, wd, md, vd)
    ids, _ = g.soft_assign(Xd, wd, md, vd, top_m=top_m, r_threshold=thr)
    idx = IVFIndex(K, ids, Xd)
    torch.cuda.synchronize()
    g.close()
    return X, md.cpu().numpy(), ids.cpu().numpy(), idx


@pytest.mark.parametrize("N,K,D", [(5000, 16, 16), (20000, 64, 128), (4099, 7, 16)])
def test_build_matches_oracle(N, K, D):
    X, C, ids, idx = _index(N, K, D, seed=31)
    off, ent = IVF.build(ids, K)
    np.testing.assert_array_equal(idx.offsets.cpu().numpy(), off)
    assert int(idx.n_entries.item()) == len(ent)
    np.testing.assert_array_equal(idx.entries[:len(ent)].cpu().numpy(), ent)


@pytest.mark.parametrize("nprobe,k", [(1, 10), (3, 10), (16, 32), (2, 1)])
def test_search_matches_oracle(nprobe, k):
    X, C, ids, idx = _index(6000, 16, 16, seed=32)
    Q = synth.generate("c1", 300, seed=33)
    out_i, out_d, dco = idx.search(torch.from_numpy(C).cuda(), Q.cuda(), nprobe, k)
    torch.cuda.synchronize()
    off, ent = IVF.build(ids, 16)
    ri, rd, rdco = IVF.search(Q.numpy(), C, off, ent, X.numpy(), nprobe, k)
    np.testing.assert_array_equal(out_i.cpu().numpy(), ri)
    np.testing.assert_array_equal(out_d.cpu().numpy(), rd)
    np.testing.assert_array_equal(dco.cpu().numpy(), rdco)


def test_search_high_dim_many_clusters():
    X, C, ids, idx = _index(20000, 64, 128, seed=34)
    Q = synth.generate("table1", 64, seed=35)
    out_i, out_d, dco = idx.search(torch.from_numpy(C).cuda(), Q.cuda(), 8, 10)
    torch.cuda.synchronize()
    off, ent = IVF.build(ids, 64)
    ri, rd, rdco = IVF.search(Q.numpy(), C, off, ent, X.numpy(), 8, 10)
    np.testing.assert_array_equal(out_i.cpu().numpy(), ri)
    np.testing.assert_array_equal(dco.cpu().numpy(), rdco)
    np.testing.assert_array_equal(out_d.cpu().numpy(), rd)
