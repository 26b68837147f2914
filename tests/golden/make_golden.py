"""Writes the golden fixtures of this directory from the oracle alone (no CUDA).

    python tests/golden/make_golden.py

tiny_em.json     one EM step (diagonal and isotropic) and the top-2 soft assignment of a
                 hand-written 2-D mixture, per "Flash-GMM: A Memory-Efficient Kernel for
                 Scalable Soft Clustering", §2 (E-step, Eqs. (1)-(3)) and §4.3 (top-2 with
                 r > tau); expected values from oracle/gmm_oracle.py.
tiny_kmeans.json one Lloyd iteration and a k-means++ seeding with fixed draws of the same
                 points (§4.4 and the initialisation appendix); expected values from
                 oracle/kmeans_oracle.py.
The inputs are written by hand below; nothing here is measured.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import gmm_oracle as O  # noqa: E402
from oracle import kmeans_oracle as KM  # noqa: E402

X = [[-2.0, -1.5], [-1.8, -2.2], [-2.5, -1.9], [-1.2, -1.0], [0.1, 0.3], [0.4, -0.2],
     [-0.3, 0.2], [0.9, 0.8], [2.1, 1.9], [2.6, 2.4], [1.9, 2.8], [3.0, 2.2]]
W = [0.3, 0.3, 0.4]
MU = [[-2.0, -2.0], [0.0, 0.0], [2.0, 2.0]]
VAR_DIAG = [[0.5, 0.4], [1.0, 0.6], [0.7, 0.9]]
VAR_SPH = [0.5, 0.8, 0.7]


def em_case(var, cov):
    r = O.em_step(np.array(X), np.array(W), np.array(MU), np.array(var), cov, 1e-6)
    ids, resp = O.soft_assign(np.array(X), np.array(W), np.array(MU), np.array(var), cov,
                              top_m=2, r_threshold=0.1)
    return {"var_in": var, "weights": r.weights.tolist(), "means": r.means.tolist(),
            "variances": r.variances.tolist(), "loglik": r.loglik, "logZ": r.logZ.tolist(),
            "soft_ids": ids.tolist(), "soft_resp": resp.tolist()}


def main():
    em = {"X": X, "weights_in": W, "means_in": MU, "reg_covar": 1e-6,
          "top_m": 2, "r_threshold": 0.1,
          "diag": em_case(VAR_DIAG, O.COV_DIAG), "spherical": em_case(VAR_SPH, O.COV_SPHERICAL)}
    with open(os.path.join(HERE, "tiny_em.json"), "w") as f:
        json.dump(em, f, indent=1)
    Xf = np.array(X, dtype=np.float32)
    C0 = np.array([[-1.0, -1.0], [0.5, 0.5], [2.5, 2.5], [9.0, 9.0]], dtype=np.float32)
    Cn, a, counts, inertia = KM.lloyd_step(Xf, C0)
    u = [0.61, 0.07, 0.93]
    idx, _ = KM.kmeanspp(Xf, 4, 5, u)
    km = {"X": X, "C0": C0.tolist(), "centroids": Cn.tolist(), "assign": a.tolist(),
          "counts": counts.tolist(), "inertia": inertia, "seed_first": 5, "seed_u": u,
          "seed_idx": idx.tolist()}
    with open(os.path.join(HERE, "tiny_kmeans.json"), "w") as f:
        json.dump(km, f, indent=1)


if __name__ == "__main__":
    main()
