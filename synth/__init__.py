"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module draws data and initial parameters only.  It holds none of the EM
arithmetic (no densities, no responsibilities, no statistics), so that the
oracle and the CUDA path share nothing but their inputs.

Workloads (stand-ins for the paper's shapes; the SIFT1M / Deep10M / GloVe-100
corpora of "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
Clustering", §4.4, are not used and nothing of them is reproduced):

  c1      N=10,000, D=16, K=16: 16 equal-weight components, means U[-5,5]^D,
          per-dim σ U[0.5,1.5].
  table1  D=128, K=1024 (Table 1's shape): means N(0, 4·I), per-dim σ
          log-uniform[0.3, 3], Dirichlet(1) weights, labels ~ Categorical.
  ivf     D=128, 20,000 latent anisotropic clusters (means N(0, 4·I), per-dim σ
          log-uniform[0.1, 2]) with Zipf(1.1) sizes fixed by largest remainder.
  border  table1 generator with K_true components plus a fraction of points
          drawn midway between two distinct component means.

Initial parameters for every workload: K distinct data rows chosen by a seeded
permutation as means, unit variances, equal weights 1/K.

Large N is generated on the target device in fixed-size chunks; each chunk has
its own seed so a prefix of the data does not depend on the total N.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

CHUNK = 1 << 20


@dataclass
class MixtureSpec:
    D: int
    K_true: int
    mean_kind: str            # "uniform5" | "normal2"
    sigma_lo: float
    sigma_hi: float
    sigma_kind: str           # "uniform" | "loguniform"
    weights_kind: str         # "equal" | "dirichlet1" | "zipf"
    zipf_s: float = 1.1
    border_frac: float = 0.0


SPECS = {
    "c1": MixtureSpec(16, 16, "uniform5", 0.5, 1.5, "uniform", "equal"),
    "table1": MixtureSpec(128, 1024, "normal2", 0.3, 3.0, "loguniform", "dirichlet1"),
    "ivf": MixtureSpec(128, 20000, "normal2", 0.1, 2.0, "loguniform", "zipf"),
    "border": MixtureSpec(960, 256, "normal2", 0.3, 3.0, "loguniform", "dirichlet1",
                          border_frac=0.10),
}


def spec(name: str, **over) -> MixtureSpec:
    s = SPECS[name]
    return MixtureSpec(**{**s.__dict__, **over})


def _cpu_gen(seed: int, salt: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed((seed * 1_000_003 + salt) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def latent_components(sp: MixtureSpec, seed: int):
    """True means [K_true, D], per-dim sigmas [K_true, D], weights [K_true] (CPU, fp64)."""
    g = _cpu_gen(seed, 1)
    K, D = sp.K_true, sp.D
    if sp.mean_kind == "uniform5":
        mu = torch.rand(K, D, generator=g, dtype=torch.float64) * 10.0 - 5.0
    else:
        mu = torch.randn(K, D, generator=g, dtype=torch.float64) * 2.0
    u = torch.rand(K, D, generator=g, dtype=torch.float64)
    if sp.sigma_kind == "uniform":
        sig = sp.sigma_lo + (sp.sigma_hi - sp.sigma_lo) * u
    else:
        sig = torch.exp(math.log(sp.sigma_lo) + (math.log(sp.sigma_hi) - math.log(sp.sigma_lo)) * u)
    if sp.weights_kind == "equal":
        w = torch.full((K,), 1.0 / K, dtype=torch.float64)
    elif sp.weights_kind == "dirichlet1":
        e = -torch.log(torch.rand(K, generator=g, dtype=torch.float64).clamp_min(1e-300))
        w = e / e.sum()
    else:  # zipf over rank j = 1..K
        r = torch.arange(1, K + 1, dtype=torch.float64)
        w = r.pow(-sp.zipf_s)
        w = w / w.sum()
    return mu, sig, w


def _exact_counts(w: torch.Tensor, N: int) -> torch.Tensor:
    """Largest-remainder apportionment of N points to weights w."""
    q = w * N
    base = torch.floor(q).to(torch.int64)
    rem = N - int(base.sum())
    if rem > 0:
        frac = q - base.to(torch.float64)
        idx = torch.argsort(frac, descending=True, stable=True)[:rem]
        base[idx] += 1
    return base


def generate(name_or_spec, N: int, seed: int = 0, device="cpu", dtype=torch.float32,
             out: torch.Tensor | None = None):
    """Return X [N, D] (torch, on ``device``) drawn from the workload's mixture.

    dtype float32 or bfloat16 (bf16 is the fp32 draw rounded to nearest once).
    ``out`` may be a preallocated [N, D] tensor of that dtype on ``device``.
    """
    sp = spec(name_or_spec) if isinstance(name_or_spec, str) else name_or_spec
    device = torch.device(device)
    mu, sig, w = latent_components(sp, seed)
    mu_d, sig_d = mu.to(device, torch.float32), sig.to(device, torch.float32)
    X = out if out is not None else torch.empty(N, sp.D, device=device, dtype=dtype)
    assert X.shape == (N, sp.D) and X.dtype == dtype
    if sp.weights_kind == "zipf":
        counts = _exact_counts(w, N)
        g = _cpu_gen(seed, 2)
        labels_all = torch.repeat_interleave(torch.arange(sp.K_true), counts)
        labels_all = labels_all[torch.randperm(N, generator=g)]
    else:
        labels_all = None
        cumw = torch.cumsum(w, 0).to(torch.float64)
        cumw[-1] = 1.0
    for c0 in range(0, N, CHUNK):
        c1 = min(N, c0 + CHUNK)
        n = c1 - c0
        gd = torch.Generator(device=device)
        gd.manual_seed((seed * 7_919 + 17 + c0 // CHUNK) & 0x7FFF_FFFF_FFFF_FFFF)
        gc = _cpu_gen(seed, 100 + c0 // CHUNK)
        if labels_all is not None:
            lab = labels_all[c0:c1]
        else:
            u = torch.rand(n, generator=gc, dtype=torch.float64)
            lab = torch.searchsorted(cumw, u, right=True).clamp_max(sp.K_true - 1)
        lab_d = lab.to(device)
        eps = torch.randn(n, sp.D, generator=gd, device=device, dtype=torch.float32)
        x = mu_d[lab_d] + sig_d[lab_d] * eps
        if sp.border_frac > 0:
            nb = int(round(sp.border_frac * n))
            if nb > 0:
                a = torch.randint(0, sp.K_true, (nb,), generator=gc)
                b = torch.randint(0, sp.K_true - 1, (nb,), generator=gc)
                b = b + (b >= a).to(b.dtype)          # b uniform over the others
                sel = torch.randperm(n, generator=gc)[:nb].to(device)
                a_d, b_d = a.to(device), b.to(device)
                mid = 0.5 * (mu_d[a_d] + mu_d[b_d])
                s = torch.sqrt(0.5 * (sig_d[a_d] ** 2 + sig_d[b_d] ** 2))
                epsb = torch.randn(nb, sp.D, generator=gd, device=device, dtype=torch.float32)
                x[sel] = mid + s * epsb
        X[c0:c1] = x.to(dtype)
    return X


def init_params(X: torch.Tensor, K: int, seed: int = 0):
    """Initial Θ: K distinct seeded rows of X as means, unit variances, π = 1/K.

    Returns float32 CPU tensors (weights [K], means [K, D], diag vars [K, D]).
    """
    N, D = X.shape
    if K > N:
        raise ValueError("K > N")
    g = _cpu_gen(seed, 3)
    idx = torch.randperm(N, generator=g)[:K].sort().values
    means = X[idx.to(X.device)].to("cpu", torch.float32).clone()
    weights = torch.full((K,), 1.0 / K, dtype=torch.float32)
    variances = torch.ones(K, D, dtype=torch.float32)
    return weights, means, variances


def uniform_points(N: int, D: int, seed: int = 0, lo=-1.0, hi=1.0):
    """Plain uniform points (edge-case tests)."""
    g = _cpu_gen(seed, 4)
    return (lo + (hi - lo) * torch.rand(N, D, generator=g, dtype=torch.float64)).to(torch.float32)
