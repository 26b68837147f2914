"""The regime the benchmark times, checked element by element against the oracle.

Table-1 generator (D = 128, K = 1024), N = 2^20 + 4099 (two chunks of the library, a
ragged tail), precision AUTO with block skipping on: after a few EM steps from the
seeded start some components sit on the CUDA-core side path (stiff), others are grey
(statistics taken on both paths), and the statistics sweep visits only a fraction of
its (point tile, component block) pairs.  The test runs GPU steps until such a step
occurs (from step 5 on), then compares that step teacher-forced: the oracle runs one
step from the same input parameters over all N points (rows sharded over the host's
cores, tests/_pool_oracle.py) and the new weights, means, variances, the per-point
log Z and the log-likelihood must agree within the parity tolerances.
"""
import numpy as np
import pytest
import torch

import synth
from tests._cmp import compare_step
from tests._pool_oracle import host_cores, teacher_forced_step

pytestmark = pytest.mark.gpu


def test_table1_k1024_steady_state_auto_block_skip():
    import ivf_quantizer_b200 as q
    N, D, K = (1 << 20) + 4099, 128, 1024
    X = synth.generate("table1", N, seed=21, device="cuda")
    w0, mu0, var0 = synth.init_params(X, K, seed=21)
    g = q.GMM(K, D, precision=q.PREC_AUTO)
    g.set_block_skip(True)
    wd, md, vd = g.new_params(w0, mu0, var0)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    lz = torch.empty(N, dtype=torch.float32, device="cuda")
    checked = None
    infos = []
    for t in range(12):
        before = (wd.cpu().numpy().copy(), md.cpu().numpy().copy(), vd.cpu().numpy().copy())
        g.step(X, wd, md, vd, loglik=ll, logz=lz)
        info = g.last_step_info()
        infos.append(info)
        g.check_status()
        if (t >= 5 and info["path"] == q.PREC_FP16X3 and info["n_stiff"] > 0
                and info["n_grey"] > 0 and 0 <= info["skip_pairs"] < info["skip_pairs_all"]):
            checked = (t, before, info)
            break
    assert checked is not None, infos
    t, (w_in, m_in, v_in), info = checked
    print("checked step", t, info, "host cores", host_cores())
    ref = teacher_forced_step(X.cpu().double().numpy(), w_in, m_in, v_in)
    out = compare_step((wd.cpu().numpy(), md.cpu().numpy(), vd.cpu().numpy()), ref,
                       X.cpu().numpy(), logz_gpu=lz.cpu().numpy(), loglik_gpu=float(ll.item()))
    print(out)
    # the step really covered small components (the regime the side path and the grey
    # rule exist for) and the comparison included them
    assert np.sum((ref.Nk >= 1) & (ref.Nk < 8)) > 0
    g.close()
