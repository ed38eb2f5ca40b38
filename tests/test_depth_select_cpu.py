"""Host logic of depth selection (looped_transformer_self_b200.depth_select)
against the oracle's independent restatement of the LoopSpec page's section
2.4 (Eqs. 7, 8, 11) and its integer constraint."""
import numpy as np
import pytest

from looped_transformer_self_b200 import depth_select as DS
from oracle import depth as Dp


def test_envelope_matches_oracle():
    rng = np.random.default_rng(11)
    for _ in range(20):
        r = np.arange(1, 11)
        m = rng.uniform(0.05, 1.0) * r ** -rng.uniform(0.2, 2.0) * np.exp(rng.normal(0, 0.3, 10))
        m[rng.integers(0, 10)] = 0.0
        a, b = DS.envelope(r.tolist(), m.tolist())
        oa, ob = Dp.fit_envelope(r, m)
        assert a == pytest.approx(oa, rel=1e-9) and b == pytest.approx(ob, rel=1e-9)
    with pytest.raises(ValueError):
        DS.envelope([1, 2], [0.3, 0.0])


@pytest.mark.parametrize("R", list(range(2, 41)))
def test_pairs_and_ranking_match_oracle(R):
    assert DS.candidate_pairs(R) == Dp.feasible_pairs(R)
    for alpha, beta in [(1.03, 0.175), (0.6, 0.4), (2.0, 0.05)]:
        assert DS.ranked_pairs(alpha, beta, R) == Dp.rank_pairs(alpha, beta, R)


def test_eq8_and_bound_match_oracle():
    rng = np.random.default_rng(12)
    for _ in range(50):
        a, b, R = rng.uniform(0.3, 2.5), rng.uniform(0.01, 1.0), int(rng.integers(4, 64))
        assert DS.eq8(a, b, R) == pytest.approx(Dp.optimal_depths(a, b, R), rel=1e-12)
        d1, d2 = rng.uniform(1, 5), rng.uniform(5, 30)
        assert DS.loop_step_bound(d1, d2, R, a, b) == pytest.approx(
            Dp.cost_bound(d1, d2, R, a, b), rel=1e-12)


def test_default_depths():
    assert DS.default_depths(4) == [1, 2, 3]
    assert DS.default_depths(32) == list(range(1, 11))
