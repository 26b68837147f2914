"""The seeded input recipe (synth/): the workloads' stated structure, determinism, and
the properties the parity tests and the bench rely on.  CPU only."""
import math

import torch

import synth


def test_latent_components_follow_the_recipe():
    mu, sig, w = synth.latent_components(synth.spec("c1"), seed=0)
    assert mu.shape == (16, 16) and float(mu.min()) >= -5 and float(mu.max()) <= 5
    assert float(sig.min()) >= 0.5 and float(sig.max()) <= 1.5
    assert torch.allclose(w, torch.full((16,), 1 / 16, dtype=torch.float64))

    mu, sig, w = synth.latent_components(synth.spec("table1"), seed=0)
    assert mu.shape == (1024, 128)
    assert abs(float(mu.std()) - 2.0) < 0.05                 # means N(0, 4 I)
    assert float(sig.min()) >= 0.3 and float(sig.max()) <= 3.0
    ls = torch.log(sig)                                      # log-uniform sigma
    assert abs(float(ls.mean()) - 0.5 * (math.log(0.3) + math.log(3.0))) < 0.02
    assert abs(float(w.sum()) - 1) < 1e-12 and float(w.min()) > 0

    mu, sig, w = synth.latent_components(synth.spec("ivf"), seed=0)
    assert mu.shape == (20000, 128)
    assert float(sig.min()) >= 0.1 and float(sig.max()) <= 2.0
    assert bool((w[1:] <= w[:-1]).all())                    # Zipf by rank
    assert abs(float(w[0] / w[1]) - 2 ** 1.1) < 1e-9


def test_exact_counts_is_largest_remainder():
    w = torch.tensor([0.5, 0.3, 0.2], dtype=torch.float64)
    assert synth._exact_counts(w, 10).tolist() == [5, 3, 2]
    c = synth._exact_counts(w, 11)          # 5.5, 3.3, 2.2 -> remainders .5 .3 .2
    assert int(c.sum()) == 11 and c.tolist() == [6, 3, 2]
    _, _, wz = synth.latent_components(synth.spec("ivf"), seed=1)
    cz = synth._exact_counts(wz, 123_457)
    assert int(cz.sum()) == 123_457
    assert bool(((cz.double() - wz * 123_457).abs() < 1).all())


def test_generation_is_seeded_and_prefix_stable():
    a = synth.generate("table1", 3000, seed=5)
    b = synth.generate("table1", 3000, seed=5)
    c = synth.generate("table1", 3000, seed=6)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert a.dtype == torch.float32 and a.shape == (3000, 128)
    # a prefix does not depend on the total N (chunk-wise seeds)
    assert torch.equal(synth.generate("c1", 700, seed=2), synth.generate("c1", 1500, seed=2)[:700])
    bf = synth.generate("table1", 3000, seed=5, dtype=torch.bfloat16)
    assert torch.equal(bf, a.to(torch.bfloat16))             # the fp32 draw rounded once


def test_points_sit_near_their_components():
    # each c1 point lies within a few sigma of its nearest true mean
    X = synth.generate("c1", 4000, seed=3).double()
    mu, sig, _ = synth.latent_components(synth.spec("c1"), seed=3)
    z = ((X[:, None, :] - mu[None]) / sig[None]) ** 2        # [N, 16, D]
    best = z.sum(-1).min(1).values
    assert float(best.mean()) < 16 * 1.3                      # chi-square with 16 dof


def test_border_points_share_two_components():
    """About 10% of the border shape's points are drawn midway between two distinct
    components: they fit a midpoint better than any component, unlike the points of the
    same mixture without border points."""
    def midway_fraction(frac):
        sp = synth.spec("border", D=16, K_true=6, border_frac=frac)
        X = synth.generate(sp, 4000, seed=4).double()
        mu, sig, _ = synth.latent_components(sp, seed=4)
        comp = ((X[:, None, :] - mu[None]) / sig[None]).pow(2).sum(-1).min(1).values
        best_mid = torch.full((X.shape[0],), float("inf"), dtype=torch.float64)
        for a in range(6):
            for b in range(6):
                if a != b:
                    m = 0.5 * (mu[a] + mu[b])
                    sd = torch.sqrt(0.5 * (sig[a] ** 2 + sig[b] ** 2))
                    best_mid = torch.minimum(best_mid, ((X - m) / sd).pow(2).sum(-1))
        return float((best_mid < comp).double().mean())
    with_border, without = midway_fraction(0.10), midway_fraction(0.0)
    assert abs((with_border - without) - 0.10) < 0.03, (with_border, without)


def test_init_params_are_distinct_rows():
    X = synth.generate("table1", 5000, seed=7)
    w, mu, var = synth.init_params(X, 300, seed=7)
    assert w.shape == (300,) and torch.allclose(w, torch.full((300,), 1 / 300))
    assert torch.equal(var, torch.ones(300, 128))
    rows = {tuple(r.tolist()) for r in X}
    assert all(tuple(m.tolist()) in rows for m in mu)
    assert len({tuple(m.tolist()) for m in mu}) == 300
    w2, mu2, _ = synth.init_params(X, 300, seed=7)
    assert torch.equal(mu, mu2)
