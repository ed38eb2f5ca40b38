"""Pins of the oracle's readout processing, residual operator, cascade and RNG.

Each test checks the oracle against something other than itself: published
known-answer vectors, closed forms, brute force on tiny vocabularies, exact
enumeration of the cascade's law, and chi-square tests of sampled draws.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats

from oracle import sampling as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_dist(rng, V, sparsity=0.0):
    w = rng.gamma(0.5, size=V)
    if sparsity:
        w[rng.random(V) < sparsity] = 0.0
        if w.sum() == 0:
            w[rng.integers(V)] = 1.0
    return w / w.sum()


# -- Philox -----------------------------------------------------------------


def test_philox_known_answer_vectors():
    """Random123's published Philox-4x32-10 vectors (tests/golden)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = S.philox4x32_10(np.array([v[:4]], dtype=np.uint64), (v[4], v[5]))[0]
        assert [int(x) for x in out] == v[6:10]


def test_philox_uniformity():
    b = S.bits(12345, 7, S.PROP1, 200_000)
    counts = np.bincount((b >> np.uint32(24)).astype(np.int64), minlength=256)
    assert scipy.stats.chisquare(counts).pvalue > 1e-3
    u = (b >> np.uint32(8)).astype(np.float64) * 2.0 ** -24
    assert 0.0 <= u.min() and u.max() < 1.0
    assert abs(u.mean() - 0.5) < 0.005


def test_streams_are_distinct():
    a = S.bits(1, 5, S.PROP1, 64)
    assert not np.array_equal(a, S.bits(1, 6, S.PROP1, 64))
    assert not np.array_equal(a, S.bits(1, 5, S.PROP2, 64))
    assert not np.array_equal(a, S.bits(2, 5, S.PROP1, 64))
    assert not np.array_equal(a, S.bits(1 + (1 << 32), 5, S.PROP1, 64))


# -- readout processing -------------------------------------------------------


def test_greedy_is_onehot_lowest_index_on_ties():
    z = np.array([0.0, 3.0, 1.0, 3.0])
    assert list(S.process(z, 0.0, 1.0)) == [0.0, 1.0, 0.0, 0.0]


def test_softmax_with_temperature_matches_library():
    rng = np.random.default_rng(0)
    z = rng.normal(size=50) * 4
    for T in (0.5, 1.0, 2.0):
        np.testing.assert_allclose(S.process(z, T, 1.0), scipy.special.softmax(z / T),
                                   rtol=1e-13, atol=1e-16)


def test_top_p_worked_examples():
    z = np.log(np.array([0.5, 0.3, 0.2]))
    np.testing.assert_allclose(S.process(z, 1.0, 0.6), [0.625, 0.375, 0.0], atol=1e-12)
    np.testing.assert_allclose(S.process(z, 1.0, 0.5), [1.0, 0.0, 0.0], atol=1e-12)
    np.testing.assert_allclose(S.process(z, 1.0, 0.81), [0.5, 0.3, 0.2], atol=1e-12)
    # tie at the boundary is kept whole
    z = np.log(np.array([0.4, 0.3, 0.3]))
    np.testing.assert_allclose(S.process(z, 1.0, 0.5), [0.4, 0.3, 0.3], atol=1e-12)


def test_top_p_brute_force_over_subsets():
    """Kept set = the smallest 'upper set' {j : p_j >= t} with mass >= top_p,
    found by enumerating all subsets of a small vocabulary."""
    rng = np.random.default_rng(1)
    V = 9
    for trial in range(200):
        p = _rand_dist(rng, V)
        if trial % 3 == 0:  # force ties
            p[1] = p[2] = p[3]
            p /= p.sum()
        top_p = float(rng.uniform(0.05, 0.99))
        best = None
        for k in range(1, V + 1):
            for sub in itertools.combinations(range(V), k):
                s = set(sub)
                upper = all((j in s) for j in range(V) for i in s if p[j] >= p[i])
                if upper and p[list(sub)].sum() >= top_p:
                    if best is None or len(sub) < len(best):
                        best = sub
            if best is not None:
                break
        q = S.process(np.log(p), 1.0, top_p)
        assert set(np.nonzero(q)[0]) == set(best)
        np.testing.assert_allclose(q.sum(), 1.0, rtol=1e-12)


# -- residual operator (Eq. 2) ------------------------------------------------


def test_residual_zero_mass_when_equal():
    p = _rand_dist(np.random.default_rng(2), 16)
    assert S.residual(p, p) is None
    assert S.residual(p, p + 0.0) is None


def test_residual_elementwise_definition():
    rng = np.random.default_rng(3)
    for _ in range(100):
        mu, nu = _rand_dist(rng, 16), _rand_dist(rng, 16, 0.3)
        r = S.residual(mu, nu)
        pos = [max(a - b, 0.0) for a, b in zip(mu, nu)]
        tot = sum(pos)
        for v in range(16):
            assert abs(r[v] - pos[v] / tot) < 1e-15
        assert np.all(r[mu <= nu] == 0.0)


def test_race_samples_its_weights():
    """The exponential race is an exact categorical sampler (chi-square)."""
    rng = np.random.default_rng(4)
    w = _rand_dist(rng, 16, 0.2) * 7.3  # unnormalised
    n = 40_000
    counts = np.zeros(16)
    for uid in range(n):
        counts[S.race(w, 99, uid, S.RES)] += 1
    exp = w / w.sum() * n
    m = exp > 0
    assert np.all(counts[~m] == 0)
    assert scipy.stats.chisquare(counts[m], exp[m]).pvalue > 0.01


def test_residual_draws_match_brute_force_residual():
    """Draws from p (-) q follow the brute-force normalised max(0, p - q)."""
    rng = np.random.default_rng(5)
    p, q = _rand_dist(rng, 16), _rand_dist(rng, 16)
    bf = np.array([max(a - b, 0.0) for a, b in zip(p, q)])
    bf /= bf.sum()
    n = 40_000
    counts = np.zeros(16)
    r = S.residual(p, q)
    for uid in range(n):
        counts[S.race(r, 3, uid, S.RES)] += 1
    m = bf > 0
    assert np.all(counts[~m] == 0)
    assert scipy.stats.chisquare(counts[m], bf[m] * n).pvalue > 0.01


# -- cascade (Eqs. 3-6) --------------------------------------------------------


@pytest.mark.parametrize("mode", ["gated", "ungated", "masked", "single"])
def test_cascade_commits_exactly_the_target(mode):
    """Exact enumeration: the committed law equals p_R for every mode."""
    rng = np.random.default_rng(6)
    for trial in range(60):
        V = 8
        pR = _rand_dist(rng, V, 0.2 if trial % 2 else 0.0)
        q1 = _rand_dist(rng, V, 0.2 if trial % 3 else 0.0)
        pd2 = _rand_dist(rng, V)
        if trial % 4 == 0:
            pd2 = 0.5 * (pd2 + pR)
        law, _ = S.cascade_law(pR, q1, None if mode == "single" else pd2,
                               "gated" if mode == "single" else mode)
        np.testing.assert_allclose(law, pR, atol=1e-12)


def test_double_rejection_bounds():
    """Section 2.3: without the gate P(no proposal committed) <= TV(p_d2, p_R);
    with the gate <= 2 TV(p_d2, p_R)."""
    rng = np.random.default_rng(7)
    worst_u, worst_g = 0.0, 0.0
    for _ in range(3000):
        V = 6
        pR = _rand_dist(rng, V)
        q1 = _rand_dist(rng, V)
        pd2 = 0.7 * pR + 0.3 * _rand_dist(rng, V)
        tv = 0.5 * np.abs(pd2 - pR).sum()
        _, fu = S.cascade_law(pR, q1, pd2, "ungated")
        _, fg = S.cascade_law(pR, q1, pd2, "gated")
        assert fu <= tv + 1e-12
        assert fg <= 2 * tv + 1e-12
        worst_u, worst_g = max(worst_u, fu / tv), max(worst_g, fg / tv)
    assert worst_g > 1.0  # the gated bound really needs its factor 2 sometimes


def test_gated_second_proposal_never_repeats_the_first():
    """Section 3.4: when the gate opens, p_d2 (-) q1 is zero at x1."""
    rng = np.random.default_rng(8)
    for _ in range(500):
        q1, pd2 = _rand_dist(rng, 12), _rand_dist(rng, 12)
        x1 = int(rng.integers(12))
        if S.gate_open(pd2, q1, x1):
            assert S.residual(pd2, q1)[x1] == 0.0


def test_greedy_gate_is_deep_argmax_change():
    rng = np.random.default_rng(9)
    for _ in range(200):
        z1, z2 = rng.normal(size=10), rng.normal(size=10)
        q1, pd2 = S.process(z1, 0, 1), S.process(z2, 0, 1)
        x1 = int(np.argmax(z1))
        assert S.gate_open(pd2, q1, x1) == (int(np.argmax(z2)) != x1)


def test_greedy_cascade_reduces_to_argmax():
    rng = np.random.default_rng(10)
    for uid in range(300):
        zR, z1, z2 = rng.normal(size=6), rng.normal(size=6), rng.normal(size=6)
        if uid % 3 == 0:
            z1 = zR
        pR, q1, pd2 = (S.process(z, 0, 1) for z in (zR, z1, z2))
        x1 = int(np.argmax(z1))
        gate = S.gate_open(pd2, q1, x1)
        x2 = int(np.argmax(z2)) if gate else -1
        q2 = S.residual(pd2, q1) if gate else None
        x, src, fb = S.verify(pR, x1, q1, gate, x2, q2, 0, uid)
        assert x == int(np.argmax(zR)) and fb == 0
        assert src == (1 if x == x1 else 2 if (gate and x == x2) else 0)


def test_no_rejection_when_draft_equals_target():
    rng = np.random.default_rng(11)
    p = _rand_dist(rng, 16)
    for uid in range(500):
        x1 = S.race(p, 1, uid, S.PROP1)
        x, src, fb = S.verify(p, x1, p, False, -1, None, 1, uid)
        assert (x, src, fb) == (x1, 1, 0)


def _v16_readouts():
    """p_d1, p_d2, p_R of the 16-token tiny model at the last prompt position,
    T = 1 with top-p 0.9 (truncated) and 1.0."""
    import synthetic as syn
    from oracle import decode as D
    from oracle.model import LoopedModel
    cfg = syn.MODELS["tiny16"]
    prompt = syn.prompt_for("tiny16", 8)
    m = LoopedModel(cfg, syn.make_weights(cfg), 16)
    zs = D.prefill(D.OracleRows(m), prompt, cfg.R, [2, 3, 4], keep_logits=True)
    return {r: zs[(len(prompt) - 1, r)] for r in (2, 3, 4)}


@pytest.mark.parametrize("top_p", [0.9, 1.0])
def test_cascade_draws_match_target_chisquare(top_p):
    """10^5 seeded committed tokens of the cascade on a 16-token vocabulary
    (proposals at depths 2 and 3, target at depth 4 of the tiny model) follow
    p_R: chi-square p > 0.01."""
    z = _v16_readouts()
    pR, q1, pd2 = (S.process(z[r], 1.0, top_p) for r in (4, 2, 3))
    n = 100_000
    counts = np.zeros(16)
    opened = 0
    for uid in range(n):
        x1 = S.race(q1, 2, uid, S.PROP1)
        gate = S.gate_open(pd2, q1, x1)
        q2 = S.residual(pd2, q1) if gate else None
        x2 = S.race(q2, 2, uid, S.PROP2) if gate else -1
        opened += gate
        x, _, fb = S.verify(pR, x1, q1, gate, x2, q2, 2, uid)
        assert fb == 0
        counts[x] += 1
    m = pR > 0
    assert np.all(counts[~m] == 0)
    assert scipy.stats.chisquare(counts[m], pR[m] * n).pvalue > 0.01
    assert 0 < opened < n
