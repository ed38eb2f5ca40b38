"""Law of the oracle's pipelined sampled decoder, end to end.

The method is lossless: with sampling, the committed sequence has exactly
the law of full-depth autoregressive decoding from the processed p_R
(LoopSpec page, section 1; section 2.2, Eqs. 2-4; section 2.3, Eqs. 5-6, the
cascade over two proposals).  Here the whole SpecDecoder -- prefill, the
pipelined schedule, proposals at d1 and d2, the gate, the cascade verify and
the re-rooting -- runs over a scripted model whose readouts depend on the
prefix AND the depth, and the joint law of the first two decoded tokens is
compared with the exact autoregressive joint, enumerated over a 16-token
vocabulary (256 bins; bins expecting fewer than 5 draws are pooled).

A second, white-box pin checks what each proposal step stores: the gate is
Eq. 6 evaluated on the branch's own depth-d2 readout against its own q1, q2
is the normalised residual p_d2 (-) q1 (or the masked / ungated variants),
and x2 lies in q2's support.  (A decoder that draws x2 from one q2 and
verifies it against another, or verifies with q1 and q2 swapped, breaks the
joint law; a wrong gate input does not break the law -- the cascade is exact
for any gate decision -- so the gate is pinned directly.)
"""
import zlib

import numpy as np
import pytest
import scipy.stats

from oracle import decode as D
from oracle import sampling as S

V = 16
PROMPT = [3, 11]


class PrefixRows:
    """Readout logits that depend on the prefix and the depth:
    z(prefix, r) = base(prefix) + (R - r) * spread * noise(prefix, r), each a
    seeded N(0, 1) vector keyed by a hash of its arguments, so shallow
    readouts disagree with full depth by a depth-dependent amount."""

    def __init__(self, R, spread=0.55, scale=1.4):
        self.R, self.spread, self.scale = R, spread, scale
        self.memo = {}

    def _vec(self, key):
        h = zlib.crc32(np.asarray(key, dtype=np.int64).tobytes())
        return np.random.default_rng(h).normal(size=V)

    def z(self, prefix, r):
        k = (tuple(int(t) for t in prefix), r)
        if k not in self.memo:
            base = self.scale * self._vec(k[0] + (-1,))
            self.memo[k] = base + (self.R - r) * self.spread * self._vec(k[0] + (r,))
        return self.memo[k]

    def prelude(self, prefix, pos, slots):
        return None

    def iterate(self, h, r, prefix, pos, slots):
        return None

    def readout(self, h, r, prefix, pos, slots, head=True):
        return self.z(prefix, r).copy() if head else None


def exact_ar_joint(rows, R, T, top_p):
    """P(t1, t2) of full-depth AR decoding after the prompt, summed over the
    prefill's first token x0: sum_x0 pR(x0 | P) pR(t1 | P x0) pR(t2 | P x0 t1)."""
    pr = lambda pre: S.process(rows.z(pre, R), T, top_p)
    J = np.zeros((V, V))
    p0 = pr(PROMPT)
    for x0 in np.nonzero(p0)[0]:
        p1 = pr(PROMPT + [x0])
        for t1 in np.nonzero(p1)[0]:
            J[t1] += p0[x0] * p1[t1] * pr(PROMPT + [x0, t1])
    return J


def sampled_joint(rows, R, d1, d2, second, T, top_p, n):
    counts = np.zeros((V, V))
    agg = D.Stats()
    for seed in range(n):
        sd = D.SpecDecoder(rows, PROMPT, R, d1, d2, 2, T, top_p, seed, 64, second=second,
                           keep_trace=False)
        res = sd.run()
        counts[res.tokens[1], res.tokens[2]] += 1
        for f in ("n_first", "n_second", "n_fallback", "gate_checks", "gate_opens",
                  "resid_fallback"):
            setattr(agg, f, getattr(agg, f) + getattr(sd.stats, f))
    return counts, agg


def pooled_chisquare(counts, expect_p, n):
    """Chi-square p-value after pooling every bin expecting < 5 draws into one."""
    e = expect_p.ravel() * n
    c = counts.ravel()
    assert np.all(c[e == 0] == 0), "a draw landed on a zero-probability pair"
    small = (e < 5) & (e > 0)
    big = e >= 5
    obs = list(c[big]) + ([c[small].sum()] if small.any() else [])
    exp = list(e[big]) + ([e[small].sum()] if small.any() else [])
    return scipy.stats.chisquare(obs, exp).pvalue


CASES = [
    # (d1, d2, R, second, top_p)
    (1, 2, 4, "gated", 1.0),
    (2, 3, 4, "gated", 0.9),
    (1, 2, 4, "ungated", 0.9),
    (2, 3, 4, "ungated", 1.0),
    (1, 2, 4, "masked", 1.0),
    (2, 3, 4, "masked", 0.9),
]


@pytest.mark.parametrize("d1,d2,R,second,top_p", CASES)
def test_first_two_tokens_follow_the_exact_ar_joint(d1, d2, R, second, top_p):
    """10^4 seeds of the full pipelined decoder (T = 1): the joint of decoded
    tokens 1 and 2 matches the exact AR joint (pooled chi-square p > 0.01), and
    every cascade outcome occurred (first accepted, second accepted, drawn
    from the residual) with the gate both opening and staying closed."""
    rows = PrefixRows(R)
    n = 10_000
    J = exact_ar_joint(rows, R, 1.0, top_p)
    assert abs(J.sum() - 1.0) < 1e-12
    counts, st = sampled_joint(rows, R, d1, d2, second, 1.0, top_p, n)
    assert counts.sum() == n
    assert pooled_chisquare(counts, J, n) > 0.01
    assert st.n_first > 0 and st.n_second > 0 and st.n_fallback > 0
    assert st.resid_fallback == 0
    if second == "gated":
        assert 0 < st.gate_opens < st.gate_checks
    elif second == "ungated":
        assert st.gate_opens > 0


def test_single_proposal_follows_the_exact_ar_joint():
    rows = PrefixRows(4)
    n = 10_000
    J = exact_ar_joint(rows, 4, 1.0, 1.0)
    counts, st = sampled_joint(rows, 4, 1, 0, "gated", 1.0, 1.0, n)
    assert pooled_chisquare(counts, J, n) > 0.01
    assert st.n_second == 0 and st.n_first > 0 and st.n_fallback > 0


@pytest.mark.parametrize("second", ["gated", "ungated", "masked"])
def test_proposal_steps_store_the_defined_gate_and_second_proposal(second):
    """After every step, each branch that has just reached d2 holds: gate =
    Eq. 6 on ITS depth-d2 readout and ITS q1 = processed p_d1 (gated), or the
    ablation's fixed rule; q2 = normalised residual p_d2 (-) q1 (gated,
    ungated) or p_d2 with x1 removed (masked); x2 in q2's support; x1 in
    q1's support.  Readouts are recomputed here from the script, not read
    from the decoder."""
    R, d1, d2, T, top_p = 4, 1, 2, 1.0, 0.9
    rows = PrefixRows(R)
    checked = opened = 0
    for seed in range(300):
        sd = D.SpecDecoder(rows, PROMPT, R, d1, d2, 4, T, top_p, seed, 64, second=second,
                           keep_trace=False)
        while not sd.done():
            sd.step()
            for b in sd.branches.values():
                if b.depth != d2 or b.retiring or b.x1 < 0:
                    continue
                pre = sd.prefix_of(b)
                q1 = S.process(rows.z(pre, d1), T, top_p)
                pd2 = S.process(rows.z(pre, d2), T, top_p)
                np.testing.assert_array_equal(b.q1, q1)
                assert q1[b.x1] > 0
                if second == "gated":
                    want_gate = pd2[b.x1] < q1[b.x1]
                    want_q2 = S.residual(pd2, q1) if want_gate else None
                elif second == "ungated":
                    want_q2 = S.residual(pd2, q1)
                    want_gate = want_q2 is not None
                else:
                    want_q2 = S.masked_second(pd2, b.x1)
                    want_gate = want_q2 is not None
                assert b.gate == want_gate
                if want_gate:
                    r = np.maximum(pd2 - q1, 0.0) if second != "masked" else np.where(
                        np.arange(V) == b.x1, 0.0, pd2)
                    np.testing.assert_allclose(b.q2, r / r.sum(), rtol=0, atol=1e-15)
                    np.testing.assert_array_equal(b.q2, want_q2)
                    assert b.q2[b.x2] > 0
                    opened += 1
                else:
                    assert b.x2 < 0
                checked += 1
    assert checked > 300 and opened > 0
