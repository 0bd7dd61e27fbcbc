"""Pins of the oracle's estimate and top-p stages: the invariants of nucleus
selection (p = 1 keeps all, a one-hot spike keeps one, uniform weights keep
ceil(p n), retained mass >= p and minimal), exhaustive subset search on tiny
inputs, the closed-form kept fraction of Gaussian logits, and exact logits when
the keys lie on the quantisation grid."""
import itertools
import math

import numpy as np
import pytest
from scipy.stats import norm

import oracle as O


def test_p_one_keeps_every_candidate():
    rng = np.random.default_rng(0)
    w = O.softmax_weights(rng.standard_normal(1000) * 5)
    sel, theta, k, *_ = O.topp_select(w, 1.0)
    assert k == 1000 and sel.tolist() == list(range(1000))
    assert theta == w.min()


def test_one_hot_spike_keeps_one():
    rng = np.random.default_rng(1)
    for p in (0.5, 0.85, 0.99, 0.999999):
        l = rng.standard_normal(4096)
        l[1234] = 60.0
        sel, theta, k, *_ = O.topp_select(O.softmax_weights(l), p)
        assert sel.tolist() == [1234] and k == 1


@pytest.mark.parametrize("n", [1, 7, 100, 4096])
@pytest.mark.parametrize("p", [0.1, 0.5, 0.85, 0.9, 0.99])
def test_uniform_keeps_ceil_pn(n, p):
    w = O.softmax_weights(np.zeros(n))
    sel, theta, k, *_ = O.topp_select(w, p)
    expect = math.ceil(p * n - 1e-9)
    assert k == expect
    assert sel.tolist() == list(range(expect))   # ties go to the lowest positions


def test_mass_at_least_p_and_minimal():
    rng = np.random.default_rng(2)
    for trial in range(200):
        n = int(rng.integers(1, 3000))
        w = O.softmax_weights(rng.standard_normal(n) * rng.uniform(0.1, 4))
        p = float(rng.uniform(0.05, 0.999))
        sel, theta, k, order, cs = O.topp_select(w, p)
        mass = w[sel].sum()
        assert mass >= p - O.MASS_EPS - 1e-13
        smallest = w[sel].min()
        assert smallest == theta
        assert mass - smallest < p - O.MASS_EPS + 1e-13
        # every unselected weight is <= theta
        mask = np.ones(n, bool)
        mask[sel] = False
        assert np.all(w[mask] <= theta)


def test_exhaustive_subsets_tiny():
    rng = np.random.default_rng(3)
    for trial in range(150):
        n = int(rng.integers(1, 11))
        w = O.softmax_weights(rng.standard_normal(n) * 2)
        p = float(rng.uniform(0.05, 0.99))
        sel, *_ = O.topp_select(w, p)
        best = None
        for r in range(1, n + 1):
            feas = [c for c in itertools.combinations(range(n), r) if w[list(c)].sum() >= p]
            if feas:
                best = max(feas, key=lambda c: w[list(c)].sum())
                break
        assert sorted(best) == sel.tolist()


def test_gaussian_kept_fraction_closed_form():
    # weights proportional to exp(sigma z), z ~ N(0,1): the mass above z0 is
    # P(Z > z0 - sigma), so the kept fraction at p is 1 - Phi(sigma + Phi^-1(1 - p))
    rng = np.random.default_rng(4)
    n = 400000
    for sigma, p in ((1.0, 0.85), (1.7, 0.85), (0.5, 0.7)):
        l = rng.standard_normal(n) * sigma
        sel, *_ = O.topp_select(O.softmax_weights(l), p)
        expect = 1 - norm.cdf(sigma + norm.ppf(1 - p))
        assert abs(len(sel) / n - expect) < 0.006, (sigma, p, len(sel) / n, expect)


def test_estimate_exact_on_grid_keys():
    # keys whose groups lie exactly on a power-of-two grid dequantise exactly,
    # so the estimate equals the exact attention logit q.k / sqrt(128)
    rng = np.random.default_rng(5)
    C = 64
    codes = rng.integers(0, 16, size=(C, 128))
    codes[:, ::32] = 0
    codes[:, 1::32] = 15
    zeros = rng.integers(-8, 8, size=(C, 4)).astype(np.float64) * 0.5
    scale = 2.0 ** rng.integers(-4, 1, size=(C, 4))
    k = (np.repeat(zeros, 32, 1) + np.repeat(scale, 32, 1) * codes).astype(np.float16)
    assert np.array_equal(k.astype(np.float64),
                          np.repeat(zeros, 32, 1) + np.repeat(scale, 32, 1) * codes)
    q = rng.standard_normal((3, 128)).astype(np.float16)
    c, s, z = O.quantize_keys(k)
    l = O.estimate_logits(q, c, s, z)
    ref = np.array([[math.fsum(float(q[h, j]) * float(k[i, j]) for j in range(128)) / math.sqrt(128)
                     for h in range(3)] for i in range(C)])
    np.testing.assert_allclose(l, ref, rtol=0, atol=1e-12)


def test_group_weights_properties():
    rng = np.random.default_rng(6)
    l = rng.standard_normal((500, 4)) * 2
    w = O.group_weights(l)
    assert abs(w.sum() - 1) < 1e-12
    np.testing.assert_allclose(O.group_weights(l[:, :1]), O.softmax_weights(l[:, 0]), atol=1e-15)
    same = np.repeat(l[:, :1], 4, 1)
    np.testing.assert_allclose(O.group_weights(same), O.softmax_weights(l[:, 0]), atol=1e-15)
    # a constant shift of one head's logits does not change its normalised weights
    l2 = l.copy()
    l2[:, 2] += 37.0
    np.testing.assert_allclose(O.group_weights(l2), w, atol=1e-15)
    # the group weight is the average, so it is between the per-head extremes
    per = np.stack([O.softmax_weights(l[:, h]) for h in range(4)], 1)
    assert np.all(w <= per.max(1) + 1e-15) and np.all(w >= per.min(1) - 1e-15)


def test_group_weights_hand_worked_example():
    """Hand-derived group weights and group top-p (tests/golden/
    group_weights_worked_example.json): separates the mean of the per-head
    normalised weights from the softmax of the mean logits."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "group_weights_worked_example.json")))
    l = np.log(np.array(g["logits_ln"], np.float64))
    w = O.group_weights(l)
    np.testing.assert_allclose(w, np.array(g["expected_weights_num84"]) / 84.0, rtol=0, atol=1e-15)
    for case in g["topp_cases"]:
        sel = O.topp_select(w, case["p"])[0]
        assert sel.tolist() == case["keep"], case
    # the wrong reading keeps a different set at p = 0.40
    wrong = O.softmax_weights(l.mean(1))
    assert O.topp_select(wrong, 0.40)[0].tolist() == g["mean_logit_reading_keep_at_0_40"]
    assert O.topp_select(w, 0.40)[0].tolist() != g["mean_logit_reading_keep_at_0_40"]
