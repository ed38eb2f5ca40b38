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


class _FakeDecoder:
    """Stands in for binding.Decoder in greedy calibration: prefill returns
    fixed readout logits [n][n_tags][V] (CPU tensors)."""

    def __init__(self, cfg, dec, z):
        self.cfg, self.dec, self.z = cfg, dec, z

    def prefill(self, tokens, argmax=False, logits=False):
        import torch
        assert logits and len(tokens) == self.z.shape[0]
        return 0, None, torch.from_numpy(self.z.copy())


def test_greedy_calibration_matches_oracle():
    """copyloop.calibrate (greedy) on fixed readout logits picks the oracle's
    tau from the same scores and acceptances (oracle.copy.prompt_calibration)."""
    import synthetic as syn
    cfg = syn.MODELS["tiny"]
    dec = syn.DECODES["tiny_greedy"]  # readout depths 2, 3, 4
    rng = np.random.default_rng(8)
    base = list(rng.integers(0, 12, size=30))
    prompt = np.array(base + base[:20] + base[5:25], dtype=np.int32)
    P, V = len(prompt), cfg.vocab
    z = rng.normal(size=(P, 3, V)).astype(np.float32)
    # make full depth agree with the copied continuation at some positions
    nxt = {t: int(prompt[t + 1]) for t in range(P - 1)}
    for t in range(P - 1):
        if rng.uniform() < 0.5:
            z[t, 2, nxt[t]] += 8.0
            z[t, 0, nxt[t]] += rng.uniform(0.0, 6.0)
    got = CL.calibrate(_FakeDecoder(cfg, dec, z), prompt)
    tau, scores, acc = CP.prompt_calibration(prompt, z[:, 0].astype(np.float64),
                                             z[:, 2].astype(np.float64), 4, 16, 64, greedy=True)
    assert got["proposals"] == len(scores) > 10
    assert got["tau"] == pytest.approx(tau, rel=1e-12)
    assert got["admitted"] == int(np.sum(np.asarray(scores) >= tau))
