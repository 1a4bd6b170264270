"""Pins of the oracle's alpha-entmax against facts fixed outside the oracle.

alpha-entmax is defined (Peters, Niculae & Martins 2019; used by DashAttention
under "Stage 1: entmax chunk routing") as the maximiser of
<p, z> + H_alpha(p) over the probability simplex.  Each test checks the
oracle against something it does not compute itself: the variational
definition through a generic constrained optimiser, a brute-force search over
supports with a generic root finder, the sparsemax closed form (alpha = 2,
Martins & Astudillo 2016), the two-element closed forms, the softmax limit
alpha -> 1, and the invariances of the definition.
"""

import itertools
import math

import numpy as np
import pytest
from scipy.optimize import brentq, minimize

from oracle.dash_oracle import entmax, entmax_threshold, entmax_threshold_bisect

ALPHAS = [1.25, 1.5, 1.75, 2.0]


def tsallis(p, alpha):
    return float(np.sum(p - p ** alpha) / (alpha * (alpha - 1.0)))


def objective(p, z, alpha):
    return float(p @ z) + tsallis(p, alpha)


@pytest.mark.parametrize("alpha", ALPHAS)
@pytest.mark.parametrize("seed", range(4))
def test_variational_definition(alpha, seed):
    """p maximises <p,z> + H_alpha(p) on the simplex (generic SLSQP cross-check)."""
    rng = np.random.default_rng(seed)
    n = 7
    z = rng.normal(size=n) * 2.0
    p, _ = entmax(z, alpha)
    res = minimize(
        lambda u: -objective(np.clip(u, 0, None), z, alpha),
        np.full(n, 1.0 / n),
        method="SLSQP",
        bounds=[(0.0, 1.0)] * n,
        constraints=[{"type": "eq", "fun": lambda u: u.sum() - 1.0}],
        options={"ftol": 1e-14, "maxiter": 1000},
    )
    assert res.success
    assert objective(p, z, alpha) >= -res.fun - 1e-10
    np.testing.assert_allclose(p, np.clip(res.x, 0, None), atol=2e-4)
    # no random point of the simplex does better
    for u in rng.dirichlet(np.ones(n) * 0.5, size=2000):
        assert objective(u, z, alpha) <= objective(p, z, alpha) + 1e-12


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("seed", range(6))
def test_brute_force_support(alpha, seed):
    """Exactly one support is self-consistent, and it is the oracle's (N <= 10)."""
    rng = np.random.default_rng(100 + seed)
    n = 6 + seed % 5
    z = rng.normal(size=n) * (1.0 + seed)
    x = (alpha - 1.0) * z
    pw = 1.0 / (alpha - 1.0)
    consistent = []
    for k in range(1, n + 1):
        for sub in itertools.combinations(range(n), k):
            xs = x[list(sub)]
            lo, hi = xs.max() - 1.0, xs.min()

            def f(t):
                return float(np.sum((xs - t) ** pw)) - 1.0

            if f(hi) >= 0.0:
                continue
            tau = brentq(f, lo, hi, xtol=1e-15, rtol=1e-15) if f(lo) > 0 else lo
            outside = np.delete(x, list(sub))
            if np.all(outside <= tau):
                consistent.append((set(sub), tau))
    assert len(consistent) == 1
    support, tau = consistent[0]
    p, tau_o = entmax(z, alpha)
    assert set(np.nonzero(p > 0)[0]) == support
    assert abs(tau_o - tau) < 1e-12


def sparsemax_textbook(z):
    """Martins & Astudillo (2016), sort-based sparsemax."""
    zs = np.sort(z)[::-1]
    cs = np.cumsum(zs)
    ks = np.arange(1, len(z) + 1)
    kz = ks[1.0 + ks * zs > cs].max()
    tau = (cs[kz - 1] - 1.0) / kz
    return np.maximum(z - tau, 0.0)


@pytest.mark.parametrize("seed", range(10))
def test_sparsemax_closed_form(seed):
    rng = np.random.default_rng(200 + seed)
    z = rng.normal(size=1 + seed * 37) * (0.1 + seed)
    p, _ = entmax(z, 2.0)
    np.testing.assert_allclose(p, sparsemax_textbook(z), atol=1e-13)


def test_alpha_to_one_is_softmax():
    rng = np.random.default_rng(3)
    z = rng.normal(size=12)
    sm = np.exp(z - z.max())
    sm /= sm.sum()
    errs = []
    for eps in (1e-2, 1e-3, 1e-4):
        p, _ = entmax(z, 1.0 + eps)
        errs.append(np.abs(p - sm).max())
    assert errs[-1] < 1e-3
    # error shrinks about linearly in alpha - 1
    assert 5.0 < errs[0] / errs[1] < 20.0
    assert 5.0 < errs[1] / errs[2] < 20.0


@pytest.mark.parametrize("alpha", ALPHAS)
def test_simplex_and_invariances(alpha):
    rng = np.random.default_rng(4)
    z = rng.normal(size=50) * 3.0
    p, _ = entmax(z, alpha)
    assert np.all(p >= 0.0)
    assert abs(p.sum() - 1.0) < 1e-12
    # shift invariance
    p2, _ = entmax(z + 7.25, alpha)
    np.testing.assert_allclose(p2, p, atol=1e-12)
    # permutation equivariance
    perm = rng.permutation(len(z))
    p3, _ = entmax(z[perm], alpha)
    np.testing.assert_allclose(p3, p[perm], atol=1e-12)
    # uniform input gives the uniform distribution
    pu, _ = entmax(np.full(9, 0.3), alpha)
    np.testing.assert_allclose(pu, np.full(9, 1.0 / 9.0), atol=1e-12)
    # monotone: larger score never gets smaller probability
    order = np.argsort(z)
    assert np.all(np.diff(p[order]) >= -1e-15)


@pytest.mark.parametrize("alpha", ALPHAS)
def test_one_hot_condition(alpha):
    """p is one-hot iff x_(1) - x_(2) >= 1 on the x = (alpha-1) z scale."""
    for gap, one_hot in ((1.0 + 1e-6, True), (1.0 - 1e-3, False)):
        z = np.array([0.2, -0.4, 0.0, 0.2 + gap / (alpha - 1.0)])
        p, _ = entmax(z, alpha)
        assert (np.count_nonzero(p) == 1) == one_hot
        if one_hot:
            assert p[3] == 1.0


@pytest.mark.parametrize("t", [-1.9, -1.0, -0.3, 0.0, 0.45, 1.2, 1.99])
def test_two_element_closed_forms(t):
    # alpha = 1.5: sqrt(p1) - sqrt(1 - p1) = t / 2 for |t| < 2
    p, _ = entmax(np.array([t, 0.0]), 1.5)
    a = (t / 2.0 + math.sqrt(2.0 - t * t / 4.0)) / 2.0
    assert abs(p[0] - a * a) < 1e-13
    # alpha = 2: p1 = clip((t + 1) / 2, 0, 1)
    p, _ = entmax(np.array([t, 0.0]), 2.0)
    assert abs(p[0] - min(1.0, max(0.0, (t + 1.0) / 2.0))) < 1e-13
    # general alpha: (alpha-1)(z1-z2) = p1^(alpha-1) - p2^(alpha-1) when both > 0
    for alpha in (1.25, 1.75):
        p, _ = entmax(np.array([t * 0.3, 0.0]), alpha)
        assert np.all(p > 0)
        lhs = (alpha - 1.0) * t * 0.3
        assert abs(lhs - (p[0] ** (alpha - 1.0) - p[1] ** (alpha - 1.0))) < 1e-12


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_bisection_agrees_with_sort(alpha):
    rng = np.random.default_rng(5)
    for n in (1, 2, 17, 511, 2047):
        x = (alpha - 1.0) * rng.normal(size=n) * 0.3
        t1 = entmax_threshold(x, alpha)
        t2 = entmax_threshold_bisect(x, alpha)
        assert abs(t1 - t2) < 1e-12
