"""fgmm_em_step_host / fgmm_em_partial_host: X streamed from host memory through two
device staging buffers must give bit-identical results to the same step on a device
copy of X (the device path is itself checked against the oracle elsewhere)."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _handle(K, D, prec):
    import ivf_quantizer_b200 as q
    g = q.GMM(K, D)
    g.set_precision({"fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO}[prec])
    return g


def _steps(g, X, w, mu, var, n_steps):
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(X.shape[0], dtype=torch.float32, device="cuda")
    lls = []
    for _ in range(n_steps):
        g.step(X, wd, md, vd, loglik=ll, logz=lz)
        lls.append(float(ll.item()))
    torch.cuda.synchronize()
    assert g.status() == 0
    return wd, md, vd, lz, lls


@pytest.mark.parametrize("prec", ["fp32", "fp16x3", "auto"])
def test_host_stream_equals_device_across_chunks(prec):
    import ivf_quantizer_b200 as q
    N = q.CHUNK_POINTS * 2 + 4321                       # three chunks, ragged tail
    X = synth.generate("c1", N, seed=7)
    w, mu, var = synth.init_params(X, 16, seed=7)
    # host rows with a stride wider than D (strided copies), pinned
    wide = torch.zeros(N, 20, dtype=torch.float32).pin_memory()
    wide[:, :16] = X
    Xh = wide[:, :16]
    a = _steps(_handle(16, 16, prec), X.cuda(), w, mu, var, 2)
    b = _steps(_handle(16, 16, prec), Xh, w, mu, var, 2)
    for ta, tb in zip(a[:4], b[:4]):
        assert torch.equal(ta, tb)
    assert a[4] == b[4]


def test_host_stream_auto_redo_and_pageable_memory():
    """AUTO steps that move collapsing components to the side path (the device path
    decision is read back before each optional pass), from pageable host memory."""
    X = synth.generate("table1", 3000, seed=2)
    w, mu, var = synth.init_params(X, 256, seed=2)
    a = _steps(_handle(256, 128, "auto"), X.cuda(), w, mu, var, 3)
    b = _steps(_handle(256, 128, "auto"), X.contiguous(), w, mu, var, 3)
    for ta, tb in zip(a[:4], b[:4]):
        assert torch.equal(ta, tb)
    assert a[4] == b[4]


def test_host_partial_matches_device_partial_and_staging_is_kept():
    import ivf_quantizer_b200 as q
    X = synth.generate("c1", 50_000, seed=3)
    w, mu, var = synth.init_params(X, 16, seed=3)
    g = _handle(16, 16, "fp32")
    wd, md, vd = g.new_params(w, mu, var)
    Xp = X.pin_memory()
    s_dev = g.partial(X.cuda(), wd, md, vd)
    s_host = g.partial(Xp, wd, md, vd)              # first host call makes the staging buffers
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    s_host2 = g.partial(Xp, wd, md, vd)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.equal(s_dev, s_host) and torch.equal(s_host, s_host2)
    assert g.status() == 0
    np.testing.assert_equal(s_dev.numel(), g.stats_len)
    g.close()
