"""GPU parity of the k-means warm start against the oracle (oracle/kmeans_oracle.py):
assignments, counts and seeding indices bit-exact (both sides decide in the same fixed
precision), centroids and inertia within the fp32 / fp64 summation tolerances."""
import numpy as np
import pytest
import torch

import synth
from oracle import kmeans_oracle as KM

pytestmark = pytest.mark.gpu


def _handle(K, D):
    import ivf_quantizer_b200 as q
    return q.GMM(K, D)


def _lloyd(X, C0):
    g = _handle(C0.shape[0], X.shape[1])
    Xd = X.cuda().contiguous() if X.dtype != torch.bfloat16 else X.cuda()
    C = torch.as_tensor(C0, dtype=torch.float32).cuda().contiguous()
    a = torch.empty(X.shape[0], dtype=torch.int32, device="cuda")
    cnt = torch.empty(C0.shape[0], dtype=torch.int64, device="cuda")
    inertia = torch.zeros(1, dtype=torch.float64, device="cuda")
    g.kmeans_step(Xd, C, assign=a, counts=cnt, inertia=inertia)
    torch.cuda.synchronize()
    assert g.status() == 0
    g.close()
    return C.cpu().numpy(), a.cpu().numpy(), cnt.cpu().numpy(), float(inertia.item())


def _check_lloyd(Xf32, C0):
    C, a, cnt, inertia = _lloyd(torch.as_tensor(Xf32), C0)
    Cr, ar, cr, ir = KM.lloyd_step(Xf32, C0)
    np.testing.assert_array_equal(a, ar)
    np.testing.assert_array_equal(cnt, cr)
    scale = np.maximum(np.abs(Cr), 1e-3)
    assert np.max(np.abs(C - Cr) / scale) <= 2e-7
    assert abs(inertia - ir) <= 1e-12 * abs(ir)


@pytest.mark.parametrize("gen,N,K", [("c1", 5000, 16), ("table1", 3000, 64), ("c1", 777, 100)])
def test_lloyd_step_matches_oracle(gen, N, K):
    X = synth.generate(gen, N, seed=11)
    C0 = X[torch.randperm(N, generator=torch.Generator().manual_seed(1))[:K]].numpy()
    _check_lloyd(X.numpy(), C0)


def test_lloyd_step_across_chunks_with_ties_and_empty_clusters():
    import ivf_quantizer_b200 as q
    N = q.CHUNK_POINTS + 3333
    X = synth.generate("c1", N, seed=12).numpy()
    C0 = X[:12].copy()
    C0[5] = C0[2]                      # duplicate centroid: index 2 must win every tie
    C0[7] = 1e4                        # far away: stays empty and keeps its centroid
    _check_lloyd(X, C0)


def test_lloyd_bf16_input_and_reproducibility():
    X = synth.generate("table1", 2500, seed=13).to(torch.bfloat16)
    Xf = X.float().numpy()
    C0 = Xf[:32].copy()
    C, a, cnt, inertia = _lloyd(X, C0)
    C2, a2, _, inertia2 = _lloyd(X, C0)
    assert np.array_equal(C, C2) and np.array_equal(a, a2) and inertia == inertia2
    Cr, ar, cr, ir = KM.lloyd_step(Xf, C0)
    np.testing.assert_array_equal(a, ar)
    np.testing.assert_array_equal(cnt, cr)
    assert abs(inertia - ir) <= 1e-12 * abs(ir)


@pytest.mark.parametrize("gen,N,K,first", [("c1", 5000, 16, 17), ("table1", 6000, 32, 0),
                                           ("c1", 9000, 8, 8999)])
def test_kmeanspp_seeding_matches_oracle_exactly(gen, N, K, first):
    X = synth.generate(gen, N, seed=14)
    u = np.random.default_rng(5).random(K - 1)
    g = _handle(K, X.shape[1])
    C, idx = g.kmeans_seed(X.cuda(), first, u)
    torch.cuda.synchronize()
    assert g.status() == 0
    g.close()
    idx_ref, C_ref = KM.kmeanspp(X.numpy(), K, first, u)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    np.testing.assert_array_equal(C.cpu().numpy(), C_ref)


def test_seeding_then_lloyd_iterations_match_oracle():
    X = synth.generate("c1", 4000, seed=15)
    K = 16
    u = np.random.default_rng(6).random(K - 1)
    g = _handle(K, 16)
    Xd = X.cuda()
    C, _ = g.kmeans_seed(Xd, 3, u)
    for _ in range(5):
        g.kmeans_step(Xd, C)
    torch.cuda.synchronize()
    g.close()
    _, C0 = KM.kmeanspp(X.numpy(), K, 3, u)
    Cr, ar, inert = KM.kmeans(X.numpy(), C0, 5)
    # the iterations agree up to the centroid summation order; on this well-separated
    # mixture every assignment is decisive, so the centroids stay within fp32 rounding
    np.testing.assert_allclose(C.cpu().numpy(), Cr, rtol=1e-5, atol=1e-5)
