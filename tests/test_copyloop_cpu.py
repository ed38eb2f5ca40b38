"""Host side of the copy screen's calibration (looped_transformer_self_b200.
copyloop): the threshold rule against the oracle's restatement
(oracle/copy.py).  The per-position lookup, scores and acceptances run on the
device (lt_copy_screen_scores; tests/test_copy_gpu.py)."""
import numpy as np

from looped_transformer_self_b200 import copyloop as CL
from oracle import copy as CP


def test_threshold_matches_oracle():
    rng = np.random.default_rng(4)
    for _ in range(200):
        n = int(rng.integers(0, 30))
        s = np.round(rng.uniform(0, 1, n), 2)  # ties
        a = rng.uniform(0, 1, n) if rng.uniform() < 0.5 else (rng.uniform(0, 1, n) < 0.5).astype(float)
        assert CL.threshold(s, a) == CP.calibrate_tau(s, a)
