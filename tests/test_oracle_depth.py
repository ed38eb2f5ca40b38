"""Pins of the depth-selection oracle (LoopSpec page, section 2.4, Eqs. 7, 8
and 11; section 3.1, Fig. 3 right) against facts that do not come from it:

* TV(p, q) is the largest gap p(A) - q(A) over events A (brute force over all
  subsets of a small vocabulary);
* a hand-worked top-p example, the greedy (T = 0) case, and the untruncated
  case against scipy's softmax;
* the envelope fit recovers an exact power law and lies on or above every
  measured mean;
* the integer pairs the page's implementation accepts, counted by hand, and the
  page's chosen (2, 8) among them;
* with residual scale 0 every depth reads out the same distribution (TV 0).
"""
import itertools

import numpy as np
import pytest
import scipy.special
import scipy.stats

import synthetic as syn
from oracle import decode as D
from oracle import depth as Dp
from oracle.model import LoopedModel


def test_total_variation_is_the_largest_event_gap():
    rng = np.random.default_rng(3)
    for _ in range(20):
        p = rng.dirichlet(np.ones(8))
        q = rng.dirichlet(np.ones(8) * 0.5)
        gap = max(abs(p[list(A)].sum() - q[list(A)].sum())
                  for k in range(9) for A in itertools.combinations(range(8), k))
        assert Dp.total_variation(p, q) == pytest.approx(gap, abs=1e-12)


def test_readout_tv_worked_top_p_example():
    # p = (.5, .3, .2): top-p 0.7 keeps {0, 1} -> (.625, .375, 0);
    # q = (.2, .3, .5): keeps {2, 1} -> (0, .375, .625).  TV = (.625 + .625) / 2.
    za = np.log([0.5, 0.3, 0.2])
    zb = np.log([0.2, 0.3, 0.5])
    assert Dp.readout_tv(za, zb, 1.0, 0.7) == pytest.approx(0.625, abs=1e-12)
    # without truncation: (.3 + 0 + .3) / 2
    assert Dp.readout_tv(za, zb, 1.0, 1.0) == pytest.approx(0.3, abs=1e-12)
    # temperature 2 flattens both by the same square root
    pa = np.sqrt([0.5, 0.3, 0.2]); pa /= pa.sum()
    pb = pa[::-1]
    assert Dp.readout_tv(za, zb, 2.0, 1.0) == pytest.approx(0.5 * np.abs(pa - pb).sum(), abs=1e-12)


def test_readout_tv_greedy_is_argmax_disagreement():
    rng = np.random.default_rng(4)
    for _ in range(50):
        za, zb = rng.normal(size=30), rng.normal(size=30)
        want = 0.0 if np.argmax(za) == np.argmax(zb) else 1.0
        assert Dp.readout_tv(za, zb, 0.0, 0.7) == want


def test_readout_tv_untruncated_matches_scipy_softmax():
    rng = np.random.default_rng(5)
    for _ in range(20):
        za, zb = 3 * rng.normal(size=100), 3 * rng.normal(size=100)
        pa, pb = scipy.special.softmax(za), scipy.special.softmax(zb)
        assert Dp.readout_tv(za, zb, 1.0, 1.0) == pytest.approx(
            np.abs(pa - pb).sum() / 2, abs=1e-12)


def test_fit_envelope_recovers_exact_power_law():
    for alpha, beta in [(1.03, 0.175), (1.08, 0.207), (0.5, 0.6)]:
        r = np.arange(1, 11)
        a, b = Dp.fit_envelope(r, beta * r ** -alpha)
        assert a == pytest.approx(alpha, rel=1e-12)
        assert b == pytest.approx(beta, rel=1e-12)


def test_fit_envelope_is_an_upper_envelope_with_least_squares_slope():
    rng = np.random.default_rng(6)
    r = np.arange(1, 11)
    m = 0.2 * r ** -0.9 * np.exp(rng.normal(scale=0.2, size=10))
    a, b = Dp.fit_envelope(r, m)
    assert a == pytest.approx(-scipy.stats.linregress(np.log(r), np.log(m)).slope, rel=1e-10)
    curve = b * r ** -a
    assert np.all(curve >= m * (1 - 1e-12))
    assert np.min(curve / m) == pytest.approx(1.0, abs=1e-12)


def test_fit_envelope_skips_zero_means():
    a, b = Dp.fit_envelope([1, 2, 3, 4], [0.4, 0.2, 0.0, 0.1])
    assert a == pytest.approx(1.0, rel=1e-12) and b == pytest.approx(0.4, rel=1e-12)
    with pytest.raises(ValueError):
        Dp.fit_envelope([1, 2, 3], [0.4, 0.0, 0.0])


def test_feasible_pairs_counted_by_hand():
    assert Dp.feasible_pairs(4) == [(1, 2), (1, 3)]
    # R = 6: d1 = 1 -> d2 in 2..5; d1 = 2 -> 4; d1 = 3 -> none (6 is not < 6)
    assert Dp.feasible_pairs(6) == [(1, 2), (1, 3), (1, 4), (1, 5), (2, 4)]
    # R = 32: 30 + 14 + 6 + 2 + 0 for d1 = 1, 2, 4, 8, 16; the page's choice is among them
    p32 = Dp.feasible_pairs(32)
    assert len(p32) == 52 and (2, 8) in p32 and (2, 9) not in p32 and (3, 6) not in p32


R32 = 32


def test_best_integer_pair_neighbours_the_continuous_optimum():
    for alpha, beta in [(1.03, 0.175), (1.08, 0.207)]:
        ranked = Dp.rank_pairs(alpha, beta, 32)
        bounds = [Dp.cost_bound(d1, d2, 32, alpha, beta) for d1, d2 in ranked]
        assert bounds == sorted(bounds)
        c1, c2 = Dp.optimal_depths(alpha, beta, 32)
        d1, d2 = ranked[0]
        assert d1 in (int(np.floor(c1)), int(np.ceil(c1)))
        # with d1 fixed, Eq. 11 is convex in d2 with its minimum where
        # beta d1^-alpha = 2 alpha beta R d2^-(alpha+1); the best d2 is a
        # neighbouring multiple of d1 of that point (which moves away from d2*
        # once d1 is rounded)
        m2 = (2 * alpha * R32 * d1 ** alpha) ** (1 / (alpha + 1))
        assert d2 in (d1 * int(np.floor(m2 / d1)), d1 * int(np.ceil(m2 / d1)))
        # the continuous point is no worse than any integer pair
        assert Dp.cost_bound(c1, c2, 32, alpha, beta) <= bounds[0]


def test_every_depth_agrees_with_zero_residual_scale():
    cfg = syn.MODELS["tiny"].replace(resid_scale=0.0)
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny")[:12]
    zs = D.prefill(D.OracleRows(LoopedModel(cfg, w, 16)), prompt, cfg.R,
                   list(range(1, cfg.R + 1)), keep_logits=True)
    tv = Dp.tv_by_depth(zs, range(len(prompt)), range(1, cfg.R), cfg.R, 1.0, 0.7)
    for r in tv:
        assert np.all(tv[r] < 1e-12)
