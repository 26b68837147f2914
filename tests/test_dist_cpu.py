"""The sharded EM iteration (ivf_quantizer_b200.dist) on CPU with world_size 2 over
gloo: the orchestration (statistics exchange, rank-ordered combination, in-place
M-step) is exercised with an engine that takes its partial statistics and its M-step
from the oracle, so the test needs no GPU.  The CUDA engine's own statistics and
M-step are checked against the same oracle functions in the GPU tests."""
import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import gmm_oracle as O


class OracleEngine:
    """partial / combine / finish with the interface of ivf_quantizer_b200.GMM, on CPU
    tensors, computed by the oracle."""

    def __init__(self, cov=O.COV_DIAG, reg=1e-6):
        self.cov, self.reg = cov, reg

    def partial(self, X, w, m, v):
        return torch.from_numpy(O.shard_statistics(X.numpy(), w.numpy(), m.numpy(), v.numpy(),
                                                   self.cov))

    def combine(self, parts):
        out = parts[0].clone()
        for p in parts[1:]:
            out += p
        return out

    def finish(self, total, w, m, v, loglik=None):
        r = O.m_step_from_statistics(total.numpy(), w.numpy(), m.numpy(), v.numpy(), self.cov,
                                     self.reg)
        w.copy_(torch.from_numpy(r.weights))
        m.copy_(torch.from_numpy(r.means))
        v.copy_(torch.from_numpy(r.variances))
        if loglik is not None:
            loglik.fill_(r.loglik)


def _data(cov):
    rng = np.random.default_rng(21)
    X = np.concatenate([rng.normal(-2, 1, (260, 3)), rng.normal(3, 0.7, (141, 3))])
    K = 3
    w = np.full(K, 1 / K)
    mu = X[[0, 5, 300]].copy()
    var = np.ones(K) if cov == O.COV_SPHERICAL else np.ones((K, 3))
    return X, w, mu, var


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, cov, mode, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=5))
    from ivf_quantizer_b200 import dist as D
    X, w, mu, var = _data(cov)
    cut = [0, 117, len(X)]                       # uneven shards
    Xs = torch.from_numpy(X[cut[rank]:cut[rank + 1]].copy())
    wt, mt, vt = (torch.from_numpy(a.copy()) for a in (w, mu, var))
    eng = OracleEngine(cov)
    try:
        if mode == "fail" and rank == 1:
            raise RuntimeError("rank 1 fails before the exchange")
        lls = []
        for _ in range(2):
            tot = D.sharded_step(eng, Xs, wt, mt, vt)
            lls.append(float(tot[-1]))
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), w=wt.numpy(), m=mt.numpy(),
                 v=vt.numpy(), ll=np.array(lls))
    except Exception as e:  # recorded for the parent; the process exits normally
        with open(os.path.join(out_dir, f"r{rank}.err"), "w") as f:
            f.write(type(e).__name__ + ": " + str(e)[:200])
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


@pytest.mark.parametrize("cov", [O.COV_DIAG, O.COV_SPHERICAL])
def test_two_rank_sharded_steps_equal_full_data_steps(tmp_path, cov):
    mp.start_processes(_worker, args=(2, _free_port(), cov, "ok", str(tmp_path)), nprocs=2,
                       join=True, start_method="spawn")
    r0, r1 = (np.load(tmp_path / f"r{r}.npz") for r in (0, 1))
    for key in ("w", "m", "v", "ll"):        # identical on both ranks, bit for bit
        np.testing.assert_array_equal(r0[key], r1[key])
    X, w, mu, var = _data(cov)
    a = O.em_step(X, w, mu, var, cov)
    b = O.em_step(X, a.weights, a.means, a.variances, cov)
    np.testing.assert_allclose(r0["m"], b.means, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r0["v"], b.variances, rtol=1e-10)
    np.testing.assert_allclose(r0["w"], b.weights, rtol=1e-10)
    np.testing.assert_allclose(r0["ll"], [a.loglik, b.loglik], rtol=1e-12)


def test_a_rank_failing_before_the_exchange_makes_the_other_fail_not_hang(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), O.COV_DIAG, "fail", str(tmp_path)),
                       nprocs=2, join=True, start_method="spawn")
    assert (tmp_path / "r1.err").read_text().startswith("RuntimeError")
    assert (tmp_path / "r0.err").exists()          # the collective raised on rank 0
    assert not (tmp_path / "r0.npz").exists()
