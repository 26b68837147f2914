"""Block skipping in the tensor-core statistics sweep (fgmm_set_block_skip).

Sweep 2 then visits only the (128-point tile, 128-component block) pairs whose
responsibilities can be non-zero at the sweep's fp16 resolution, over the points
regrouped by block.  A left-out pair adds exactly zero, so the step must agree with the
dense sweep up to the order of fp32 additions; sweep 1 (log Z, the log-likelihood) is
untouched and must agree bit for bit.  The step must also stay bitwise reproducible
from run to run and within the parity tolerances of the oracle.

Cases: well separated (one block per point), partly overlapping (a mix of one-block and
several-block points), fully overlapping (every point in every block), the largest
block count (K = 4096: 32 blocks), two blocks with a ragged tail, two chunks, AUTO.

The CUDA-core path (FGMM_PREC_FP32) skips the same way with a cut of 50 nats (each
left-out responsibility is below 2e-22): checked on the IVF shape, on D = 960 (its
statistics read the log-densities kept by sweep 1, through the reordering) and on
32 blocks.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import gmm_oracle as O
from tests._cmp import compare_step

pytestmark = pytest.mark.gpu


def _step(X, w, mu, var, skip, prec="fp16x3", steps=1):
    import ivf_quantizer_b200 as q
    K, D = mu.shape
    g = q.GMM(K, D)
    g.set_precision({"fp16x3": q.PREC_FP16X3, "auto": q.PREC_AUTO, "fp32": q.PREC_FP32}[prec])
    g.set_block_skip(skip)
    assert g.block_skip == skip
    Xd = torch.as_tensor(X).cuda().contiguous()
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(Xd.shape[0], dtype=torch.float32, device="cuda")
    for _ in range(steps):
        g.step(Xd, wd, md, vd, loglik=ll, logz=lz)
    torch.cuda.synchronize()
    assert g.status() == 0
    out = (wd.cpu().numpy(), md.cpu().numpy(), vd.cpu().numpy(), float(ll.item()), lz.cpu().numpy())
    g.close()
    return out


def _agree(a, b, X, rtol=2e-5):
    """Skip vs dense: sweep 1 bit for bit, the M-step to fp32 summation-order level.
    Means are judged against max(|mu|, per-dim data std) and variances against
    max(var, per-dim data variance): the tensor path forms the variance from raw moments
    about the global centre, so a summation-order difference of the moments shows up
    on the data's scale, not on the (possibly tiny) variance's."""
    assert a[3] == b[3]
    assert np.array_equal(a[4], b[4])
    np.testing.assert_array_equal(a[0] == 0, b[0] == 0)
    np.testing.assert_allclose(a[0], b[0], rtol=rtol, atol=1e-12)
    scale = np.maximum(np.asarray(X, np.float64).std(axis=0), 1e-30)
    dm = np.abs(a[1].astype(np.float64) - b[1]) / np.maximum(np.abs(b[1]), scale[None, :])
    assert dm.max() <= rtol, dm.max()
    dv = np.abs(a[2].astype(np.float64) - b[2]) / np.maximum(np.abs(b[2]), scale[None, :] ** 2)
    assert dv.max() <= rtol, dv.max()


def _oracle(X, w, mu, var):
    return O.em_step(np.asarray(X, np.float64), np.asarray(w, np.float64),
                     np.asarray(mu, np.float64), np.asarray(var, np.float64), 0, 1e-6)


def test_separated_table1_shape_matches_dense_and_oracle():
    N = 20_000 + 37                                   # several tiles per block, ragged tail
    X = synth.generate("table1", N, seed=3)
    w, mu, var = synth.init_params(X, 1024, seed=3)   # 8 blocks
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)
    c = _step(X, w, mu, var, True, prec="auto")
    print(compare_step(c[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=c[4], loglik_gpu=c[3]))


def test_skip_is_bitwise_reproducible():
    X = synth.generate("table1", 9_000, seed=4)
    w, mu, var = synth.init_params(X, 512, seed=4)
    a = _step(X, w, mu, var, True, steps=2)
    b = _step(X, w, mu, var, True, steps=2)
    for ta, tb in zip(a[:3], b[:3]):
        assert np.array_equal(ta, tb)
    assert a[3] == b[3]


def test_partly_overlapping_mix_of_buckets():
    """Wide initial variances put many points within the cut of several blocks."""
    X = synth.generate("table1", 12_000, seed=5)
    w, mu, var = synth.init_params(X, 640, seed=5)   # 5 blocks
    var = var * 12.0
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)
    c = _step(X, w, mu, var, True, prec="auto")
    compare_step(c[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=c[4], loglik_gpu=c[3])


def test_fully_overlapping_every_tile_dense():
    X = synth.uniform_points(7_000, 8, seed=6)
    w, mu, var = synth.init_params(X, 384, seed=6)   # 3 blocks, all within the cut
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)


def test_most_blocks_k4096():
    X = synth.generate("table1", 6_000, seed=7)[:, :64].contiguous()
    w, mu, var = synth.init_params(X, 4096, seed=7)  # 32 blocks: the largest mask
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)
    c = _step(X, w, mu, var, True, prec="auto")
    compare_step(c[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=c[4], loglik_gpu=c[3])


def test_two_blocks_ragged():
    X = synth.generate("table1", 3_005, seed=8)
    w, mu, var = synth.init_params(X, 200, seed=8)   # K = 200: 2 blocks, padded
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)
    c = _step(X, w, mu, var, True, prec="auto")
    compare_step(c[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=c[4], loglik_gpu=c[3])


def test_bf16_input():
    X = synth.generate("table1", 7_001, seed=12).to(torch.bfloat16)
    w, mu, var = synth.init_params(X.float(), 512, seed=12)
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X.float())


def test_two_chunks():
    import ivf_quantizer_b200 as q
    N = q.CHUNK_POINTS + 3_001
    X = synth.generate("c1", N, seed=9)
    X = torch.cat([X, X * 0.5 + 3.0], dim=1)         # D = 32
    w, mu, var = synth.init_params(X, 256, seed=9)
    a = _step(X, w, mu, var, True)
    b = _step(X, w, mu, var, False)
    _agree(a, b, X)


def test_auto_mode_with_skip():
    X = synth.generate("table1", 8_000, seed=10)
    w, mu, var = synth.init_params(X, 256, seed=10)
    _agree(_step(X, w, mu, var, True, prec="auto"), _step(X, w, mu, var, False, prec="auto"), X)
    # later steps, teacher-forced: the third step of one handle (AUTO carries N_k from
    # step to step) against the oracle's step from the parameters it started from
    # (free-running trajectories drift apart: EM amplifies summation-order differences)
    import ivf_quantizer_b200 as q
    g = q.GMM(256, 128)
    g.set_block_skip(True)
    Xd = X.cuda()
    wd, md, vd = g.new_params(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(X.shape[0], dtype=torch.float32, device="cuda")
    for _ in range(2):
        g.step(Xd, wd, md, vd)
    w2, m2, v2 = (t.cpu().numpy() for t in (wd, md, vd))
    g.step(Xd, wd, md, vd, loglik=ll, logz=lz)
    torch.cuda.synchronize()
    assert g.status() == 0
    compare_step((wd.cpu().numpy(), md.cpu().numpy(), vd.cpu().numpy()), _oracle(X, w2, m2, v2),
                 X.numpy(), logz_gpu=lz.cpu().numpy(), loglik_gpu=float(ll.item()))
    g.close()


def test_skip_shortens_the_statistics_sweep():
    """On the Table-1 shape (one block per point) sweep 2 runs on about 1/8 of the
    (tile, block) pairs: its device time must drop well below the dense sweep's."""
    import ivf_quantizer_b200 as q
    X = synth.generate("table1", q.CHUNK_POINTS, seed=11, device="cuda")
    w, mu, var = synth.init_params(X, 1024, seed=11)
    ms = {}
    for skip in (False, True):
        g = q.GMM(1024, 128)
        g.set_precision(q.PREC_FP16X3)
        g.set_block_skip(skip)
        wd, md, vd = g.new_params(w, mu, var)
        g.step(X, wd.clone(), md.clone(), vd.clone())
        g.profile(True)
        g.step(X, wd.clone(), md.clone(), vd.clone())
        torch.cuda.synchronize()
        ms[skip] = g.profile_read()["kernels"]["tc_stats"]["active_ms"]
        g.close()
    print(ms)
    assert ms[True] < 0.6 * ms[False]


def test_fp32_path_ivf_shape():
    X = synth.generate("ivf", 20_000 + 11, seed=13)
    w, mu, var = synth.init_params(X, 512, seed=13)   # 4 blocks of 128 components
    a = _step(X, w, mu, var, True, prec="fp32")
    b = _step(X, w, mu, var, False, prec="fp32")
    _agree(a, b, X)
    compare_step(a[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=a[4], loglik_gpu=a[3])


def test_fp32_path_high_dimension():
    X = synth.generate("border", 4_000 + 3, seed=14)
    w, mu, var = synth.init_params(X, 512, seed=14)   # D = 960: kept log-densities
    a = _step(X, w, mu, var, True, prec="fp32")
    b = _step(X, w, mu, var, False, prec="fp32")
    _agree(a, b, X)
    compare_step(a[:3], _oracle(X, w, mu, var), X.numpy(), logz_gpu=a[4], loglik_gpu=a[3])


def test_fp32_path_most_blocks_two_steps():
    X = synth.generate("table1", 6_000, seed=15)[:, :64].contiguous()
    w, mu, var = synth.init_params(X, 4096, seed=15)  # 32 blocks
    a = _step(X, w, mu, var, True, prec="fp32")
    b = _step(X, w, mu, var, False, prec="fp32")
    _agree(a, b, X)
    a2 = _step(X, w, mu, var, True, prec="fp32", steps=2)
    b2 = _step(X, w, mu, var, True, prec="fp32", steps=2)
    for ta, tb in zip(a2[:3], b2[:3]):
        assert np.array_equal(ta, tb)                  # bitwise reproducible
