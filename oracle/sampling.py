"""Readout processing, residual operator, accept cascade and random draws.

Test infrastructure only.  fp64 numpy throughout.  Follows the LoopSpec page
(liuzhao09.github.io/papers/loopspec.html):

  * section 2.1: the readout C applies temperature, optional truncation (top-p)
    and normalisation, and every intermediate readout uses the same processing
    as the target;
  * section 2.2, Eq. 2: (mu (-) nu)(v) = [mu(v) - nu(v)]_+ / sum_u [mu(u) - nu(u)]_+;
    a zero denominator means mu == nu and a rejection cannot happen;
  * section 2.2, Eqs. 3-4: x~ ~ q, accept with probability min(1, p(x~)/q(x~)),
    on rejection draw from p (-) q;
  * section 2.3, Eqs. 5-6 and the cascade: q2 = p_d2 (-) q1; the gate opens iff
    p_d2(x1) < q1(x1); at depth R verify x1 against p_R, then x2 against
    rho1 = p_R (-) q1, and after a double rejection draw from rho1 (-) q2 (gate
    closed: draw from rho1).

Readings where the pages are silent:
  * greedy (T = 0) readouts are one-hot at the argmax, lowest index on ties,
    and run through the same cascade (which then reduces to argmax compares);
  * top-p keeps every token whose probability is >= theta*, the largest value
    theta among the probabilities with sum_{p_j >= theta} p_j >= top_p (ties at
    the boundary are kept); top_p >= 1 keeps everything;
  * accept test: strict  u * q(x~) < p(x~)  with u = (bits >> 8) * 2^-24;
  * categorical draws use the exponential race x = argmin_i E_i / w_i with
    E_i = -ln v_i, v_i = ((bits_i >> 8) + 1/2) * 2^-24, weights w_i = 0 never
    chosen, lowest index on ties (Gumbel-max; unnormalised weights allowed);
  * bits come from Philox-4x32-10 (Salmon et al., "Parallel random numbers:
    as easy as 1, 2, 3", SC'11): key = (seed lo, seed hi), counter =
    (element index, uid or position, purpose, 0), first output word.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

# purposes (third counter word)
PROP1, PROP2, ACC1, ACC2, RES, AR = 1, 2, 3, 4, 5, 6

SRC_FALLBACK, SRC_FIRST, SRC_SECOND = 0, 1, 2

_M0 = np.uint64(0xD2511F53)
_M1 = np.uint64(0xCD9E8D57)
_W0 = 0x9E3779B9
_W1 = 0xBB67AE85
_MASK = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr: np.ndarray, key: Tuple[int, int]) -> np.ndarray:
    """Philox-4x32 with 10 rounds.  ctr: uint array [..., 4]; returns uint32 [..., 4]."""
    c = [np.asarray(ctr[..., i], dtype=np.uint64) & _MASK for i in range(4)]
    k0, k1 = int(key[0]) & 0xFFFFFFFF, int(key[1]) & 0xFFFFFFFF
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + _W0) & 0xFFFFFFFF
            k1 = (k1 + _W1) & 0xFFFFFFFF
        p0 = _M0 * c[0]
        p1 = _M1 * c[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK
        c = [hi1 ^ c[1] ^ np.uint64(k0), lo1, hi0 ^ c[3] ^ np.uint64(k1), lo0]
    return np.stack(c, axis=-1).astype(np.uint32)


def _key(seed: int) -> Tuple[int, int]:
    return seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF


def bits(seed: int, stream: int, purpose: int, n: int) -> np.ndarray:
    """First Philox output word for counters (i, stream, purpose, 0), i < n."""
    ctr = np.zeros((n, 4), dtype=np.uint64)
    ctr[:, 0] = np.arange(n, dtype=np.uint64)
    ctr[:, 1] = np.uint64(stream & 0xFFFFFFFF)
    ctr[:, 2] = np.uint64(purpose)
    return philox4x32_10(ctr, _key(seed))[:, 0]


def uniform(seed: int, stream: int, purpose: int) -> float:
    """u in [0, 1) from 24 bits of the counter (0, stream, purpose, 0)."""
    b = int(bits(seed, stream, purpose, 1)[0])
    return (b >> 8) * 2.0 ** -24


def race(w: np.ndarray, seed: int, stream: int, purpose: int) -> int:
    """Exponential race over non-negative weights w (need not sum to 1)."""
    w = np.asarray(w, dtype=np.float64)
    b = bits(seed, stream, purpose, w.shape[0])
    v = ((b >> np.uint32(8)).astype(np.float64) + 0.5) * 2.0 ** -24
    e = -np.log(v)
    with np.errstate(divide="ignore"):
        key = np.where(w > 0, e / np.where(w > 0, w, 1.0), np.inf)
    if not np.isfinite(key).any():
        raise ValueError("race over an all-zero weight vector")
    return int(np.argmin(key))  # first index on ties


def process(z: np.ndarray, temperature: float, top_p: float) -> np.ndarray:
    """Readout processing of logits z: temperature, top-p, normalisation."""
    z = np.asarray(z, dtype=np.float64)
    if temperature == 0.0:
        p = np.zeros_like(z)
        p[int(np.argmax(z))] = 1.0
        return p
    y = z / temperature
    e = np.exp(y - y.max())
    p = e / e.sum()
    if top_p < 1.0:
        order = np.argsort(-p, kind="stable")
        cum = np.cumsum(p[order])
        k = int(np.searchsorted(cum, top_p, side="left"))  # first k with cum[k] >= top_p
        k = min(k, p.shape[0] - 1)
        theta = p[order[k]]
        keep = p >= theta
        p = np.where(keep, p, 0.0)
        p = p / p.sum()
    return p


def residual(mu: np.ndarray, nu: np.ndarray) -> Optional[np.ndarray]:
    """(mu (-) nu) of Eq. 2; None when the positive part has zero mass."""
    pos = np.maximum(np.asarray(mu, np.float64) - np.asarray(nu, np.float64), 0.0)
    z = pos.sum()
    if z <= 0.0:
        return None
    return pos / z


def one_hot(x: int, V: int) -> np.ndarray:
    """The proposal distribution of a token that was not drawn (a copied token)."""
    q = np.zeros(V, dtype=np.float64)
    q[x] = 1.0
    return q


def gate_open(p_d2: np.ndarray, q1: np.ndarray, x1: int) -> bool:
    """Eq. 6: open iff the deeper readout lowers the first candidate's probability."""
    return bool(p_d2[x1] < q1[x1])


def verify(p_R: np.ndarray, x1: int, q1: Optional[np.ndarray], gate: bool, x2: int,
           q2: Optional[np.ndarray], seed: int, uid: int) -> Tuple[int, int, int]:
    """Cascade verification at full depth (Eqs. 3-5 and section 2.3).

    Returns (token, source, residual_fallbacks).  source: 1 = first proposal
    accepted, 2 = second proposal accepted, 0 = drawn at full depth.
    """
    fb = 0
    if x1 < 0:
        return race(p_R, seed, uid, RES), SRC_FALLBACK, 0
    u1 = uniform(seed, uid, ACC1)
    if u1 * q1[x1] < p_R[x1]:
        return x1, SRC_FIRST, 0
    rho1 = residual(p_R, q1)
    if rho1 is None:  # unreachable in exact arithmetic (p_R == q1 never rejects)
        rho1, fb = np.asarray(p_R, np.float64), 1
    if gate:
        u2 = uniform(seed, uid, ACC2)
        if u2 * q2[x2] < rho1[x2]:
            return x2, SRC_SECOND, fb
        r2 = residual(rho1, q2)
        if r2 is None:
            r2, fb = rho1, fb + 1
        return race(r2, seed, uid, RES), SRC_FALLBACK, fb
    return race(rho1, seed, uid, RES), SRC_FALLBACK, fb


def cascade_law(p_R: np.ndarray, q1: np.ndarray, p_d2: Optional[np.ndarray],
                mode: str = "gated") -> Tuple[np.ndarray, float]:
    """Exact law of the committed token under the cascade, and the probability
    that neither proposal is committed, by enumeration over x1 ~ q1 and
    x2 ~ q2 -- used to pin ``verify``.

    mode: "gated" (Eq. 5 + gate of Eq. 6), "ungated" (residual second proposal
    always opened), "masked" (ablation of section 3.4: p_d2 with x1 masked and
    renormalised, always opened).  p_d2 None: single proposal.
    """
    V = p_R.shape[0]
    law = np.zeros(V)
    p_fb = 0.0
    rho1 = residual(p_R, q1)
    for x1 in range(V):
        if q1[x1] <= 0:
            continue
        a1 = min(1.0, p_R[x1] / q1[x1])
        law[x1] += q1[x1] * a1
        rej = q1[x1] * (1.0 - a1)
        if rej <= 0.0 or rho1 is None:
            continue
        if p_d2 is None:
            q2 = None
        elif mode == "gated":
            q2 = residual(p_d2, q1) if gate_open(p_d2, q1, x1) else None
        elif mode == "ungated":
            q2 = residual(p_d2, q1)
        else:
            q2 = masked_second(p_d2, x1)
        if q2 is None:
            law += rej * rho1
            p_fb += rej
            continue
        r2 = residual(rho1, q2)
        for x2 in range(V):
            if q2[x2] <= 0:
                continue
            a2 = min(1.0, rho1[x2] / q2[x2])
            law[x2] += rej * q2[x2] * a2
            if r2 is not None:
                law += rej * q2[x2] * (1.0 - a2) * r2
                p_fb += rej * q2[x2] * (1.0 - a2)
    return law, p_fb


def masked_second(p_d2: np.ndarray, x1: int) -> Optional[np.ndarray]:
    """Non-residual second proposal (ablation, section 3.4): p_d2 with x1 masked."""
    q = np.asarray(p_d2, np.float64).copy()
    q[x1] = 0.0
    z = q.sum()
    return None if z <= 0 else q / z
