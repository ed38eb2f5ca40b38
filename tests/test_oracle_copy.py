"""Pins of the context-copy proposals (CopyLoop card: copied continuations,
screened at a shallow depth, verified at full depth; readings in
oracle/copy.py) against facts worked out by hand and against invariants:

* the lookup on hand-made sequences (longest backward match wins, the most
  recent on ties, copies stop at the committed context and at max_len);
* the screen score against scipy's softmax; the calibration's threshold on a
  hand-worked list;
* verifying a copied token with a one-hot proposal commits exactly p_R
  (enumeration and 10^5 seeded draws, chi-square);
* scripted schedules (R = 4, d1 = 1, one proposal): a copied 5-token chain
  commits in one step after its root; a full-depth disagreement inside the
  chain restarts there; a depth-1 disagreement cuts the chain at the screen;
* greedy speculative decoding with copies equals greedy full-depth decoding;
* in sampled decoding the token after a copied proposal follows p_R (a
  model whose readouts depend only on depth, 4000 seeds, chi-square).
"""
import numpy as np
import pytest
import scipy.special
import scipy.stats

import synthetic as syn
from oracle import copy as CP
from oracle import decode as D
from oracle import sampling as S
from oracle.model import LoopedModel
from scripted import ScriptedRows


def test_lookup_worked_examples():
    # one earlier occurrence of the last 4 tokens, match length 4 (limited by e = 3)
    seq = [1, 2, 3, 4, 5, 9, 1, 2, 3, 4]
    assert CP.lookup(seq, 10, 4, 16, 64) == (3, 4, [5, 9, 1, 2, 3, 4])
    # the occurrence ending at 4 matches 5 tokens back (7 1 2 3 4), the one at 10 only 4
    seq = [7, 1, 2, 3, 4, 5, 8, 1, 2, 3, 4, 6, 7, 1, 2, 3, 4]
    assert CP.lookup(seq, 17, 4, 16, 64) == (4, 5, [5, 8, 1, 2, 3, 4, 6, 7, 1, 2, 3, 4])
    # equal match lengths: the most recent occurrence
    seq = [1, 2, 3, 4, 5, 1, 2, 3, 4, 6, 1, 2, 3, 4]
    assert CP.lookup(seq, 14, 4, 16, 64) == (8, 4, [6, 1, 2, 3, 4])
    # an uncommitted last token: the copy stops at the committed context
    seq = [1, 2, 3, 4, 5, 6, 1, 2, 3, 4]
    assert CP.lookup(seq, 9, 4, 16, 64) == (3, 4, [5, 6, 1, 2, 3])
    # max_len and match_cap
    seq = [1, 2, 3, 4] + list(range(20, 40)) + [1, 2, 3, 4]
    assert CP.lookup(seq, len(seq), 4, 5, 64) == (3, 4, [20, 21, 22, 23, 24])
    seq = [5] * 12
    e, m, prop = CP.lookup(seq, 12, 4, 16, 6)
    assert (e, m, prop) == (10, 6, [5])
    # no earlier occurrence, and a match shorter than k
    assert CP.lookup([1, 2, 3, 4, 5, 6], 6, 4, 16, 64) == (-1, 0, [])
    assert CP.lookup([9, 2, 3, 4, 1, 2, 3, 4], 8, 5, 16, 64) == (-1, 0, [])


def test_screen_score_is_softmax():
    rng = np.random.default_rng(1)
    for _ in range(10):
        z = 4 * rng.normal(size=50)
        t = int(rng.integers(50))
        assert CP.screen_score(z, t) == pytest.approx(scipy.special.softmax(z)[t], rel=1e-12)


def test_calibration_worked_example():
    # gains: tau 0.9 -> +1, 0.8 -> +2, 0.3 -> +1, 0.2 -> +2; ties go to the larger tau
    assert CP.calibrate_tau([0.9, 0.8, 0.3, 0.2], [1, 1, 0, 1]) == 0.8
    assert CP.calibrate_tau([0.5, 0.4], [0, 0]) == 1.0
    assert CP.calibrate_tau([], []) == 1.0
    # fractional acceptances (sampling): keep while the mean gain stays positive
    assert CP.calibrate_tau([0.7, 0.6, 0.1], [0.9, 0.6, 0.2]) == 0.6


def test_one_hot_verification_commits_the_target():
    rng = np.random.default_rng(2)
    for _ in range(40):
        pR = rng.dirichlet(np.ones(8) * 0.7)
        s = int(rng.integers(8))
        law, _ = S.cascade_law(pR, S.one_hot(s, 8), None, "gated")
        np.testing.assert_allclose(law, pR, atol=1e-12)
    pR = rng.dirichlet(np.ones(16))
    s = 3
    n = 100_000
    counts = np.zeros(16)
    for uid in range(n):
        x, src, fb = S.verify(pR, s, S.one_hot(s, 16), False, -1, None, 5, uid)
        assert fb == 0 and (src == 1) == (x == s)
        counts[x] += 1
    assert scipy.stats.chisquare(counts, pR * n).pvalue > 0.01


# -- scripted schedules ---------------------------------------------------------

CYCLE = [10, 11, 12, 13, 14]
PROMPT = CYCLE + CYCLE + [10, 11]  # prefill commits 12


def _cycle_script(full_override=None, shallow_override=None):
    """Every depth predicts the next token of the cycle after the prefix's last
    token, except where an override (prefix length -> token) says otherwise at
    full depth (r = 4) or at depth 1."""
    def s(prefix, r):
        n = len(prefix)
        if r == 4 and full_override and n in full_override:
            return full_override[n]
        if r == 1 and shallow_override and n in shallow_override:
            return shallow_override[n]
        return CYCLE[(CYCLE.index(prefix[-1]) + 1) % 5] if prefix[-1] in CYCLE else 10
    return s


def _run(script, max_new, ar=False):
    rows = ScriptedRows(16, script)
    if ar:
        return D.decode_ar(rows, PROMPT, 4, max_new, 0.0, 1.0, 3)
    cp = D.CopyConfig(tau=0.1, table=64, reserve=4)
    return D.decode_spec(rows, PROMPT, 4, 1, 0, max_new, 0.0, 1.0, 3, 128, copy=cp)


def test_scripted_chain_commits_in_one_step():
    """Step 1: the root (prefix ends 10 11 12) copies 13 14 10 11 12 (the token
    budget of 6 allows 5 rows).  Step 4: the root verifies 13.  Step 5: all
    five chain rows are at depth 4 and commit 14 10 11 12 and the last row's
    own proposal 13."""
    sp = _run(_cycle_script(), 6)
    ar = _run(_cycle_script(), 6, ar=True)
    assert sp.tokens == ar.tokens == [12, 13, 14, 10, 11, 12, 13]
    assert sp.commit_step == [4, 5, 5, 5, 5, 5]
    assert sp.src == [1] * 6
    st = sp.stats
    assert (st.copy_chains, st.copy_rows, st.copy_cut, st.n_copy) == (1, 5, 0, 5)
    # the chain rows share every step's depth
    assert [r[3] for r in sp.trace[1]] == [2, 1, 1, 1, 1, 1]


def test_scripted_full_depth_disagreement_restarts_inside_the_chain():
    """Full depth says 7 after ... 13 14 (prefix length 15): the row at
    position 14 rejects the copied 10 in step 5, commits 7 from p_R with 10
    removed (greedy: the argmax), and the rest of the chain goes."""
    over = {15: 7}
    sp = _run(_cycle_script(full_override=over), 6)
    ar = _run(_cycle_script(full_override=over), 6, ar=True)
    assert sp.tokens == ar.tokens
    assert sp.tokens[:4] == [12, 13, 14, 7]
    assert sp.commit_step[:3] == [4, 5, 5]
    assert sp.src[:3] == [1, 1, 0]


def test_scripted_shallow_disagreement_cuts_the_chain():
    """Depth 1 says 7 after ... 13 14: in step 2 the screen of the row at
    position 14 removes the copied rows from position 15 on (three rows) and
    that row proposes 7 instead; full depth agrees with the cycle, so 7 is
    rejected later and the output still equals AR."""
    over = {15: 7}
    sp = _run(_cycle_script(shallow_override=over), 6)
    ar = _run(_cycle_script(shallow_override=over), 6, ar=True)
    assert sp.tokens == ar.tokens == [12, 13, 14, 10, 11, 12, 13]
    assert sp.stats.copy_cut == 3
    assert sp.commit_step[:2] == [4, 5]


def test_tiny_greedy_with_copies_equals_full_depth():
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny")
    n = 64
    ar = D.decode_ar(D.OracleRows(LoopedModel(cfg, w, 256)), prompt, cfg.R, n, 0.0, 1.0, 2)
    cp = D.CopyConfig(tau=0.0, table=16, reserve=7)
    sp = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, 256)), prompt, cfg.R, 2, 3, n, 0.0, 1.0,
                       2, 256, copy=cp)
    assert sp.tokens == ar.tokens
    assert sp.stats.copy_chains > 0


class _SoftRows:
    """Readouts whose logits depend only on the depth (a fixed soft p_r)."""

    def __init__(self, z_by_depth):
        self.z = z_by_depth

    def prelude(self, prefix, pos, slots):
        return None

    def iterate(self, h, r, prefix, pos, slots):
        return None

    def readout(self, h, r, prefix, pos, slots, head=True):
        return self.z[r].copy() if head else None


def test_sampled_tokens_after_a_copy_follow_p_R():
    """Sampled decoding (T = 1) with copies: prompt 1 2 3 4 5 1 2 3; when the
    first token is 4, the root's lookup copies 5 1 2 3 and the next token is
    verified with a one-hot proposal.  Over 4000 seeds the token after a
    copied proposal is distributed as p_R (chi-square p > 0.01), and copies
    were both accepted and rejected."""
    V, R = 8, 4
    rng = np.random.default_rng(9)
    zR = np.log(np.array([0.04, 0.06, 0.05, 0.05, 0.45, 0.2, 0.1, 0.05]))
    z = {r: zR + (4 - r) * 0.4 * rng.normal(size=V) for r in range(1, R + 1)}
    pR = S.process(zR, 1.0, 1.0)
    prompt = [1, 2, 3, 4, 5, 1, 2, 3]
    counts = np.zeros(V)
    copied = accepted = 0
    for seed in range(4000):
        cp = D.CopyConfig(tau=0.0, table=32, reserve=4)
        sd = D.SpecDecoder(_SoftRows(z), prompt, R, 1, 0, 2, 1.0, 1.0, seed, 64, copy=cp)
        res = sd.run()
        if res.tokens[0] != 4:
            continue
        assert sd.stats.copy_chains >= 1
        copied += 1
        accepted += res.tokens[1] == 5
        counts[res.tokens[1]] += 1
    assert copied > 1000 and 0 < accepted < copied
    assert scipy.stats.chisquare(counts, pR * copied).pvalue > 0.01
