"""Context-copy suffix proposals with shallow-depth screening (test
infrastructure only; only tests, the smoke check and the benchmark's CPU
baseline use it).

Follows the CopyLoop card (kongchang.com, "CopyLoop: training-free decoding
acceleration for looped Transformers"): candidate multi-token continuations
are copied from context that repeats; they are scored at a shallow loop depth
and only those above a threshold found by a light calibration go on to the
full-depth verification; newer blocks start while earlier ones still deepen.
The card gives no formulas.  Readings taken here (the same on the CUDA side,
which is written separately):

  * lookup: the branch's prefix is the token sequence seq[0..n-1]; L tokens of
    it are committed.  A source is an end position e with k - 1 <= e <= L - 2
    (inside the committed context and followed by a committed token) whose
    backward match with the prefix's end, m(e) = the number of t = 0, 1, ...
    (t < match_cap, t <= e) with seq[e - t] == seq[n - 1 - t] before the first
    mismatch, is at least k.  The source with the largest m(e) wins, ties going
    to the largest e (the most recent).  The proposal is seq[e + 1 ..
    min(e + max_len, L - 1)];
  * screening score of a copied token s at a readout: softmax of the logits at
    T = 1 (no truncation), taken at s -- the model's own depth-d1 probability;
    a copied token goes on only when its score is >= tau;
  * calibration of tau on the prompt: for every prompt position t (the last
    included) whose prefix has a copy proposal, score s_1 with the depth-d1
    readout of t and note whether the full-depth readout accepts it (greedy:
    its argmax is s_1; sampling: with probability p_R(s_1)); tau is the score
    threshold that maximises the sum over kept proposals of (2 accept - 1),
    i.e. a proposal is kept when it is more likely accepted than not.  No
    proposal: tau = 1 (none kept).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np


def lookup(seq: Sequence[int], L: int, k: int, max_len: int,
           match_cap: int) -> Tuple[int, int, List[int]]:
    """Copy proposal for the prefix `seq` with L committed tokens.
    Returns (e, m(e), proposal); e = -1 and [] when there is none."""
    n = len(seq)
    best_e, best_m = -1, 0
    for e in range(k - 1, L - 1):
        m = 0
        while m < match_cap and m <= e and seq[e - m] == seq[n - 1 - m]:
            m += 1
        if m >= k and m >= best_m:
            best_e, best_m = e, m
    if best_e < 0:
        return -1, 0, []
    return best_e, best_m, [int(seq[j]) for j in range(best_e + 1, min(best_e + max_len, L - 1) + 1)]


def screen_score(z: np.ndarray, tok: int) -> float:
    """softmax(z)[tok] at T = 1."""
    z = np.asarray(z, np.float64)
    e = np.exp(z - z.max())
    return float(e[tok] / e.sum())


def calibrate_tau(scores: Sequence[float], accept: Sequence[float]) -> float:
    """Threshold maximising sum over kept (score >= tau) of (2 accept - 1);
    the candidates are the observed scores (the largest such threshold wins
    ties, keeping fewer rows for the same gain)."""
    s = np.asarray(scores, np.float64)
    a = np.asarray(accept, np.float64)
    if s.size == 0:
        return 1.0
    best_tau, best_gain = 1.0, 0.0
    for tau in np.unique(s):
        gain = float((2.0 * a[s >= tau] - 1.0).sum())
        if gain > best_gain or (gain == best_gain and gain > 0 and tau > best_tau):
            best_tau, best_gain = float(tau), gain
    return best_tau


def prompt_calibration(prompt: Sequence[int], z_d1, z_R, k: int, max_len: int, match_cap: int,
                       greedy: bool, temperature: float = 1.0,
                       top_p: float = 1.0) -> Tuple[float, List[float], List[float]]:
    """tau from the prompt: z_d1[t], z_R[t] are the depth-d1 and full-depth
    readout logits of prompt position t.  Returns (tau, scores, accepts)."""
    from . import sampling as S
    scores, acc = [], []
    for t in range(len(prompt)):
        # the prefix prompt[0..t] with all of it committed (the last position
        # too: its full-depth readout exists)
        _, _, prop = lookup(prompt[:t + 1], t + 1, k, max_len, match_cap)
        if not prop:
            continue
        s1 = prop[0]
        scores.append(screen_score(z_d1[t], s1))
        if greedy:
            acc.append(1.0 if int(np.argmax(z_R[t])) == s1 else 0.0)
        else:
            acc.append(float(S.process(z_R[t], temperature, top_p)[s1]))
    return calibrate_tau(scores, acc), scores, acc
