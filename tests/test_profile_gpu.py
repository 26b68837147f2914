"""Kernel timing (fgmm_profile_*): under AUTO a step enqueues both paths and the
profile must count as active exactly the launches of the path the step took."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _profiled_step(prec_name, N, K, gen="table1", seed=0):
    import ivf_quantizer_b200 as q
    X = synth.generate(gen, N, seed=seed).cuda()
    w, mu, var = synth.init_params(X.cpu(), K, seed=seed)
    g = q.GMM(K, X.shape[1])
    g.set_precision({"auto": q.PREC_AUTO, "fp32": q.PREC_FP32, "fp16x3": q.PREC_FP16X3}[prec_name])
    wd, md, vd = g.new_params(w, mu, var)
    g.profile(True)
    g.profile_read(reset=True)
    g.step(X, wd, md, vd)
    prof = g.profile_read(reset=True)
    path = g.last_step_path()
    g.check_status()
    g.close()
    return prof, path


@pytest.mark.parametrize("N", [20000, (1 << 20) + 3000])
def test_auto_tensor_step_counts_only_tensor_launches(N):
    import ivf_quantizer_b200 as q
    chunks = -(-N // q.CHUNK_POINTS)
    prof, path = _profiled_step("auto", N, 64, seed=2)
    k = prof["kernels"]
    assert path == q.PREC_FP16X3
    # both passes of AUTO are enqueued (the redo pass returns at its gate unless the
    # variance check asked for it), the CUDA-core sweeps are enqueued and return at once
    assert k["tc_stats"]["launches"] == 2 * chunks
    assert k["tc_stats"]["active"] in (chunks, 2 * chunks)
    assert k["tc_lse"]["active"] == k["tc_stats"]["active"] == k["tc_convert"]["active"]
    assert k["stats_simt"]["launches"] == chunks and k["stats_simt"]["active"] == 0
    assert k["lse_simt"]["active"] == 0
    assert k["tc_stats"]["active_ms"] > 0
    # every kernel launch is counted: a sweep-1 region holds two (the sweep and the merge
    # of its per-block partials), every other region one
    assert prof["launches"] == sum(v["launches"] for v in k.values()) + k["tc_lse"]["launches"]


def test_fp32_step_counts_cuda_core_launches():
    import ivf_quantizer_b200 as q
    prof, path = _profiled_step("fp32", 5000, 64)
    k = prof["kernels"]
    assert path == q.PREC_FP32
    assert "tc_stats" not in k
    assert k["stats_simt"]["active"] == 1 and k["lse_simt"]["active"] == 1
