"""Failure detection without a GPU fault: the bounded device-side wait that every
tensor-core kernel uses gives up after its limit and reports FGMM_ERR_TIMEOUT (a
barrier that nothing completes), leaving the context usable."""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_expires_and_reports_timeout():
    from ivf_quantizer_b200 import _lib
    t0 = time.time()
    st = _lib.LIB.fgmm_selftest_bounded_wait(200)
    dt = time.time() - t0
    assert st == _lib.ERR_TIMEOUT
    assert dt < 30
    # the context still works afterwards
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0


def test_bounded_wait_rejects_bad_limits():
    from ivf_quantizer_b200 import _lib
    assert _lib.LIB.fgmm_selftest_bounded_wait(0) == _lib.ERR_INVALID_ARG
    assert _lib.LIB.fgmm_selftest_bounded_wait(20000) == _lib.ERR_INVALID_ARG
