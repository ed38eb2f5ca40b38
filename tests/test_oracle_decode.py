"""Pins of the oracle's decoding state machine.

* Fig. 1 of the LoopSpec page: loop-step counts 12 / 9 / 7 (tests/golden);
* section 3.4: 249 branches at most for (2, 8, 32) with unconditional forking;
* with s = 0 every depth agrees, every first proposal is accepted, commits
  come every d1 steps after the first R and gamma (Eq. 9) equals R / d1;
* gamma <= R / d1 always (section 3.2);
* lossless greedy: speculative greedy output equals full-depth greedy output
  (section 1 / 2.3);
* Eq. 8's printed optimal depths (tests/golden).
"""
import os

import numpy as np
import pytest

import synthetic as syn
from oracle import decode as D
from oracle import depth as Dp
from oracle.model import LoopedModel
from scripted import FIG1_PROMPT, ScriptedRows, fig1_script, fork_script

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    return [l.split() for l in open(os.path.join(GOLDEN, name)) if l.strip() and not l.startswith("#")]


@pytest.mark.parametrize("first_it", [True, False])
def test_fig1_loop_step_counts(first_it):
    rows = ScriptedRows(10, fig1_script(first_it))
    for mode, d1, d2, R, n, steps in _golden("fig1_loop_steps.txt"):
        d1, d2, R, n, steps = int(d1), int(d2), int(R), int(n), int(steps)
        if mode == "ar":
            res = D.decode_ar(rows, FIG1_PROMPT, R, n, 0.0, 1.0, 0)
        elif mode == "single" and not first_it:
            continue  # the left panel has every later proposal accepted
        else:
            res = D.decode_spec(rows, FIG1_PROMPT, R, d1, d2, n, 0.0, 1.0, 0, 64)
        assert res.stats.steps == steps, mode
        assert res.tokens[1:] == [3, 4, 5]  # Paris, and, it
    res = D.decode_spec(rows, FIG1_PROMPT, 4, 1, 2, 3, 0.0, 1.0, 0, 64)
    # right panel: Paris from the second proposal, "and" from the first with
    # the gate closed, "it" from the first (left) or second (the pruned "the")
    assert res.src == [2, 1, 1 if first_it else 2]


def test_max_branches_with_unconditional_forking():
    for d1, d2, R, mx in _golden("max_branches.txt"):
        d1, d2, R, mx = int(d1), int(d2), int(R), int(mx)
        res = D.decode_spec(ScriptedRows(4, fork_script(d2)), [0, 0], R, d1, d2, 60, 0.0, 1.0, 0,
                            4096, keep_trace=False)
        assert res.stats.rows_max == mx
        assert res.stats.n_first == 60 + 0 and res.stats.gate_opens > 0
        assert res.stats.table_peak >= mx


@pytest.mark.parametrize("d1,d2", [(1, 0), (2, 0), (1, 2), (2, 3)])
def test_zero_scale_accepts_every_first_proposal(d1, d2):
    cfg = syn.MODELS["tiny"].replace(resid_scale=0.0)
    m = LoopedModel(cfg, syn.make_weights(cfg), 128)
    prompt = syn.prompt_for("tiny", 8)
    n = 10
    res = D.decode_spec(D.OracleRows(m), prompt, cfg.R, d1, d2, n, 0.0, 1.0, 2, 128)
    assert res.src == [1] * n
    assert res.commit_step == [cfg.R + k * d1 for k in range(n)]
    assert res.stats.gamma(d1, d2, cfg.R) == pytest.approx(cfg.R / d1)
    assert res.stats.gate_opens == 0


def _tiny(n_slots=256):
    cfg = syn.MODELS["tiny"]
    return cfg, syn.make_weights(cfg)


def test_speculative_greedy_equals_full_depth_greedy():
    cfg, w = _tiny()
    prompt = syn.prompt_for("tiny")
    dec = syn.DECODES["tiny_greedy"]
    n = 24
    ar = D.decode_ar(D.OracleRows(LoopedModel(cfg, w, 256)), prompt, cfg.R, n, 0.0, 1.0, dec.seed)
    for d1, d2 in ((2, 3), (1, 2), (1, 0), (3, 0)):
        sp = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, 256)), prompt, cfg.R, d1, d2, n,
                           0.0, 1.0, dec.seed, 256)
        assert sp.tokens == ar.tokens
        g = sp.stats.gamma(d1, d2, cfg.R)
        assert 1.0 <= g <= cfg.R / d1 + 1e-12


def test_sampled_speculative_run_is_consistent():
    """Sampling (T = 1, top-p 0.9): every committed token has positive mass in
    the full-depth readout of its prefix, slots are never shared by two live
    branches, and committed slots are distinct."""
    cfg, w = _tiny()
    prompt = syn.prompt_for("tiny")
    dec = syn.DECODES["tiny_sample"]
    n = 16
    sp = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, 256)), prompt, cfg.R, dec.d1, dec.d2, n,
                       dec.temperature, dec.top_p, dec.seed, 256, keep_logits=True)
    seq = list(prompt) + sp.tokens
    from oracle import sampling as S
    for k, tok in enumerate(sp.tokens[1:]):
        pos = len(prompt) + k
        p = S.process(sp.logits[(pos, cfg.R)], dec.temperature, dec.top_p)
        assert p[tok] > 0
    assert len(set(sp.committed_slots)) == len(sp.committed_slots)
    for rows in sp.trace:
        slots = [s for (_, s, _, _) in rows]
        assert len(set(slots)) == len(slots)
    assert len(seq) == len(prompt) + 1 + n


def test_eq8_printed_depths():
    for a, b, R, d1, d2 in _golden("eq8_depths.txt"):
        o1, o2 = Dp.optimal_depths(float(a), float(b), float(R))
        assert round(o1, 2) == float(d1) and round(o2, 2) == float(d2)
        # it is a stationary point of the Eq. 11 bound
        f = lambda x, y: Dp.cost_bound(x, y, float(R), float(a), float(b))
        eps = 1e-6
        assert abs((f(o1 + eps, o2) - f(o1 - eps, o2)) / (2 * eps)) < 1e-5
        assert abs((f(o1, o2 + eps) - f(o1, o2 - eps)) / (2 * eps)) < 1e-5


def test_rollback_keeps_output_lossless_and_commit_branch_edits_tree():
    """Rolling back a speculative branch only discards work: greedy output is
    unchanged.  Committing a root child appends its token, re-roots on it and
    keeps only its subtree."""
    cfg, w = _tiny()
    prompt = syn.prompt_for("tiny", 16)
    n = 14
    ref = D.decode_ar(D.OracleRows(LoopedModel(cfg, w, 128)), prompt, cfg.R, n, 0.0, 1.0, 2)
    sd = D.SpecDecoder(D.OracleRows(LoopedModel(cfg, w, 128)), prompt, cfg.R, 1, 2, n, 0.0, 1.0,
                       2, 128)
    rolled = 0
    while not sd.done():
        sd.step()
        root = sd.root().uid if not sd.done() else None
        others = [u for u in sd.branches if u != root]
        if others and rolled < 3 and sd.stats.steps % 5 == 0:
            sd.rollback(max(others))
            rolled += 1
            live = [b.slot for b in sd.branches.values()]
            assert len(set(live)) == len(live) and not (set(live) & sd.free)
    assert rolled == 3 and sd.committed[len(prompt):] == ref.tokens

    sd = D.SpecDecoder(D.OracleRows(LoopedModel(cfg, w, 128)), prompt, cfg.R, 1, 2, n, 0.0, 1.0,
                       2, 128)
    for _ in range(3):
        sd.step()
    root = sd.root()
    child = sd.branches[root.child1]
    L = len(sd.committed)
    sd.commit_branch(child.uid)
    assert sd.committed[-1] == child.token and len(sd.committed) == L + 1
    assert sd.root().uid == child.uid and sd.src[-1] == 3
    assert sd.cslots[-1] == child.slot and root.slot in sd.cslots
    for b in sd.branches.values():
        if not b.retiring:
            assert b.uid == child.uid or child.uid in _ancestors(sd, b)
    # the old root had iterations left: it retires (stays until its R-th)
    assert [b.uid for b in sd.branches.values() if b.retiring] == [root.uid]
    assert root.depth < cfg.R and root.slot not in sd.free


def test_no_row_reads_a_cache_row_that_was_never_written():
    """Every cache row a row attends to was computed first, also around
    external commits (whose old root has not run all R iterations) and
    rollbacks: with unwritten rows set to NaN, every readout stays finite and
    the tokens equal those of the zero-filled run; a retiring root leaves the
    table right after its R-th iteration."""
    cfg, w = _tiny()
    prompt = syn.prompt_for("tiny", 16)

    def run(unwritten):
        sd = D.SpecDecoder(D.OracleRows(LoopedModel(cfg, w, 128, unwritten=unwritten)), prompt,
                           cfg.R, 1, 2, 14, 0.0, 1.0, 2, 128, keep_logits=True)
        commits, leave = 0, {}
        while not sd.done():
            sd.step()
            for u, s in list(leave.items()):
                if sd.stats.steps == s:
                    assert u not in sd.branches
                    del leave[u]
                else:
                    assert u in sd.branches and sd.branches[u].retiring
            if sd.done():
                break
            root = sd.root()
            if sd.stats.steps >= (3, 8, 1 << 30)[commits] and root.child1 in sd.branches:
                sd.commit_branch(root.child1)
                commits += 1
                leave[root.uid] = sd.stats.steps + cfg.R - root.depth
            elif sd.stats.steps == 6:
                others = [u for u, b in sd.branches.items() if u != root.uid and not b.retiring]
                if others:
                    sd.rollback(max(others))
        assert commits == 2 and not leave
        return sd

    a, b = run(np.nan), run(0.0)
    assert all(np.isfinite(z).all() for z in a.logits.values())
    assert a.committed == b.committed and a.src == b.src


def _ancestors(sd, b):
    out = []
    x = sd.branches.get(b.parent)
    while x is not None:
        out.append(x.uid)
        x = sd.branches.get(x.parent)
    return out
