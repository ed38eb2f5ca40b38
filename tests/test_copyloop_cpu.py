"""Host calibration of the copy screen (looped_transformer_self_b200.copyloop)
against the oracle's restatement (oracle/copy.py): first copied tokens of
every prompt prefix and the threshold rule."""
import numpy as np
import pytest

from looped_transformer_self_b200 import copyloop as CL
from oracle import copy as CP


@pytest.mark.parametrize("seed,k,cap", [(0, 4, 64), (1, 4, 6), (2, 2, 64), (3, 5, 8)])
def test_first_copies_match_oracle_lookup(seed, k, cap):
    rng = np.random.default_rng(seed)
    seq = list(rng.integers(0, 6, size=40))
    for _ in range(6):  # paste earlier spans to make long matches
        a = int(rng.integers(0, len(seq) - 8))
        seq += seq[a:a + int(rng.integers(4, 12))] + [int(rng.integers(0, 6))]
    got = CL.first_copies(seq, k, cap)
    for t in range(len(seq)):
        _, _, prop = CP.lookup(seq[:t + 1], t + 1, k, 16, cap)
        assert got.get(t) == (prop[0] if prop else None), t


def test_threshold_matches_oracle():
    rng = np.random.default_rng(4)
    for _ in range(200):
        n = int(rng.integers(0, 30))
        s = np.round(rng.uniform(0, 1, n), 2)  # ties
        a = rng.uniform(0, 1, n) if rng.uniform() < 0.5 else (rng.uniform(0, 1, n) < 0.5).astype(float)
        assert CL.threshold(s, a) == CP.calibrate_tau(s, a)
