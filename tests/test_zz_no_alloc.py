"""The allocation-free soft assignment (fgmm_soft_assign_static).

Some host programs may not call cudaMalloc at all (device memory owned by an arena
reserved up front; loops that cannot afford the allocator's implicit device
synchronisation), so they cannot create a handle.  This entry point keeps its
scratch in a fixed array inside the library instead.  The test calls it through the
C-ABI and checks it against the handle-based fgmm_soft_assign on two calls in a row
with different problem sizes (the second call finds the first call's data in the
shared array), and that device memory does not change across calls once the first
call on the device (its set-up) has run.

Collected last on purpose: when a run stops at the first failure, every other test
has already run.  Passes alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _static_assign(X, w, mu, var, K, D, cov, top_m, thr, ids, resp):
    from ivf_quantizer_b200 import _lib
    n = X.shape[0]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dt = _lib.BF16 if X.dtype == torch.bfloat16 else _lib.F32
    rc = _lib.LIB.fgmm_soft_assign_static(
        K, D, cov, ctypes.c_void_p(X.data_ptr()), dt, n, X.stride(0),
        ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(mu.data_ptr()),
        ctypes.c_void_p(var.data_ptr()), top_m, thr, ctypes.c_void_p(ids.data_ptr()),
        ctypes.c_void_p(resp.data_ptr() if resp is not None else 0), stream)
    return rc, ids, resp


def _free_bytes_stable():
    """Free device memory, read twice if the first two reads disagree (another process
    on the same GPU may allocate between them)."""
    torch.cuda.synchronize()
    a = torch.cuda.mem_get_info()[0]
    b = torch.cuda.mem_get_info()[0]
    return a if a == b else torch.cuda.mem_get_info()[0]


def _handle_assign(X, w, mu, var, K, D, cov, top_m, thr):
    import ivf_quantizer_b200 as q
    g = q.GMM(K, D, cov)
    ids, resp = g.soft_assign(X, w, mu, var, top_m=top_m, r_threshold=thr)
    torch.cuda.synchronize()
    g.close()
    return ids, resp


def _problem(name, N, K, seed, cov):
    X = synth.generate(name, N, seed=seed).cuda()
    w, mu, var = synth.init_params(X.cpu(), K, seed=seed)
    var = var * 2.0
    if cov == 1:
        var = var[:, 0].contiguous()
    return X, w.cuda(), mu.cuda(), var.cuda().contiguous()


def test_static_soft_assign_matches_handle_path_twice():
    from ivf_quantizer_b200 import _lib
    cases = [("table1", 3000, 200, 2, 0, 2, 1.0 / 200), ("c1", 5000, 16, 3, 1, 3, 0.01)]
    refs = [None, None]
    for j, (name, N, K, seed, cov, top_m, thr) in enumerate(cases):
        X, w, mu, var = _problem(name, N, K, seed, cov)
        refs[j] = (X, w, mu, var, K, X.shape[1], cov, top_m, thr,
                   _handle_assign(X, w, mu, var, K, X.shape[1], cov, top_m, thr))
    outs = [(torch.full((r[0].shape[0], r[7]), -7, dtype=torch.int32, device="cuda"),
             torch.full((r[0].shape[0], r[7]), -7.0, dtype=torch.float32, device="cuda"))
            for r in refs]
    # the first call on a device is its set-up: the library looks up the scratch array's
    # device address, and the CUDA runtime may materialise the array (lazy module
    # loading); the calls after it must not change device memory
    X0, w0, mu0, var0, K0, D0, cov0, m0, t0, _ = refs[0]
    assert _static_assign(X0, w0, mu0, var0, K0, D0, cov0, m0, t0, *outs[0])[0] == _lib.OK
    free0 = _free_bytes_stable()
    rcs = []
    for attempt in range(2):
        rcs = []
        for (X, w, mu, var, K, D, cov, top_m, thr, _), (ids, resp) in zip(refs, outs):
            rcs.append(_static_assign(X, w, mu, var, K, D, cov, top_m, thr, ids, resp)[0])
        free1 = _free_bytes_stable()
        if free1 == free0:
            break
        free0 = free1   # another process allocated in between: measure once more
    assert rcs == [_lib.OK, _lib.OK], rcs
    assert free1 == free0          # no device allocation by the calls after the set-up
    for (*_, (rid, rresp)), (ids, resp) in zip(refs, outs):
        assert torch.equal(ids.cpu(), rid.cpu())
        np.testing.assert_allclose(resp.cpu().numpy(), rresp.cpu().numpy(), rtol=1e-6, atol=0)


def test_static_soft_assign_rejects_oversize_and_bad_arguments():
    from ivf_quantizer_b200 import _lib
    X = torch.zeros(8, 4, device="cuda")
    p = torch.zeros(64, device="cuda")
    ids = torch.zeros(8, 2, dtype=torch.int32, device="cuda")
    null = ctypes.c_void_p(0)

    def call(K, D, top_m=1, thr=0.0, x=X):
        return _lib.LIB.fgmm_soft_assign_static(
            K, D, 0, ctypes.c_void_p(x.data_ptr()), _lib.F32, x.shape[0], max(D, x.stride(0)),
            ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(p.data_ptr()),
            ctypes.c_void_p(p.data_ptr()), top_m, thr, ctypes.c_void_p(ids.data_ptr()), null,
            null)

    # padded K x padded D above the fixed scratch: refused before any work is enqueued
    assert call(1 << 12, 128) == _lib.ERR_UNSUPPORTED
    assert call(_lib.STATIC_MAX_K + 1, 1) == _lib.ERR_UNSUPPORTED
    assert call(0, 4) == _lib.ERR_INVALID_ARG
    assert call(4, 4, top_m=5) == _lib.ERR_INVALID_ARG
    assert call(4, 4, thr=1.0) == _lib.ERR_INVALID_ARG


def test_static_soft_assign_bf16_null_resp_and_status_word():
    """bf16 input and resp = NULL against the handle path; an invalid variance comes back
    as ERR_INVALID_ARG from the device status word, and the next valid call returns OK
    (the word is cleared by every call)."""
    from ivf_quantizer_b200 import _lib
    X, w, mu, var = _problem("table1", 2500, 96, 4, 0)
    Xb = X.to(torch.bfloat16)
    rid, rresp = _handle_assign(Xb, w, mu, var, 96, X.shape[1], 0, 2, 0.05)
    ids = torch.full((X.shape[0], 2), -7, dtype=torch.int32, device="cuda")
    resp = torch.full((X.shape[0], 2), -7.0, dtype=torch.float32, device="cuda")
    assert _static_assign(Xb, w, mu, var, 96, X.shape[1], 0, 2, 0.05, ids, resp)[0] == _lib.OK
    assert torch.equal(ids.cpu(), rid.cpu())
    np.testing.assert_allclose(resp.cpu().numpy(), rresp.cpu().numpy(), rtol=1e-6, atol=0)
    ids2 = torch.full_like(ids, -7)
    assert _static_assign(X, w, mu, var, 96, X.shape[1], 0, 2, 0.05, ids2, None)[0] == _lib.OK
    rid32, _ = _handle_assign(X, w, mu, var, 96, X.shape[1], 0, 2, 0.05)
    assert torch.equal(ids2.cpu(), rid32.cpu())
    bad = var.clone()
    bad[3, 5] = -1.0
    assert _static_assign(X, w, mu, bad, 96, X.shape[1], 0, 2, 0.05, ids2, None)[0] == \
        _lib.ERR_INVALID_ARG
    ids3 = torch.full_like(ids, -7)
    assert _static_assign(X, w, mu, var, 96, X.shape[1], 0, 2, 0.05, ids3, None)[0] == _lib.OK
    assert torch.equal(ids3.cpu(), rid32.cpu())
