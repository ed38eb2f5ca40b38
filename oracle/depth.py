"""Depth selection of the LoopSpec page, section 2.4 (test infrastructure only).

The oracle is test infrastructure: only tests, the smoke check and the
benchmark's CPU baseline use it.

Eq. 7 bounds the mean total variation between the depth-r readout and the
target by a power law beta * r^-alpha; Eq. 11 bounds the expected serial loop
steps per committed token by d1 + beta d1^-alpha d2 + 2 beta d2^-alpha R; its
stationary point is Eq. 8:
    D = alpha^2 + alpha + 1,
    d1* = (alpha beta)^((alpha+1)/D) (2 alpha R)^(1/D),
    d2* = (alpha beta)^(alpha/D) (2 alpha R)^((alpha+1)/D).

Measurement side (section 3.1, Fig. 3 right): TV(p_r, p_R) at T = 1, top-p
0.7, averaged over token positions of a fixed prefix, for several depths r;
a power law through those means, raised until it lies on or above every one
of them, is the empirical envelope of Eq. 7 whose (alpha, beta) feed Eq. 8.
Eq. 8's point is continuous; the implementation the page describes needs
integers 1 <= d1 < d2 < R with d2 and R multiples of d1, and the page treats
the formula as the start of a search that wall-clock measurement finishes.

Readings where the page is silent:
  * the power law is fitted by least squares on (ln r, ln mean TV) for alpha;
    beta is then the smallest value for which beta r^-alpha >= every mean;
  * depths whose mean TV is 0 carry no information about the slope and are
    left out of the fit;
  * integer candidates are ranked by Eq. 11's bound (ascending; ties by d1,
    then d2).
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np

from . import sampling as S


def cost_bound(d1: float, d2: float, R: float, alpha: float, beta: float) -> float:
    """Eq. 11 right-hand side."""
    return d1 + beta * d1 ** -alpha * d2 + 2.0 * beta * d2 ** -alpha * R


def optimal_depths(alpha: float, beta: float, R: float) -> Tuple[float, float]:
    """Eq. 8: continuous stationary point of the Eq. 11 bound."""
    D = alpha * alpha + alpha + 1.0
    d1 = (alpha * beta) ** ((alpha + 1.0) / D) * (2.0 * alpha * R) ** (1.0 / D)
    d2 = (alpha * beta) ** (alpha / D) * (2.0 * alpha * R) ** ((alpha + 1.0) / D)
    return d1, d2


def total_variation(p: np.ndarray, q: np.ndarray) -> float:
    """TV(p, q) = 1/2 sum_v |p(v) - q(v)|."""
    return 0.5 * float(np.abs(np.asarray(p, np.float64) - np.asarray(q, np.float64)).sum())


def readout_tv(z_a: np.ndarray, z_b: np.ndarray, temperature: float, top_p: float) -> float:
    """TV between the processed readouts (section 2.1) of two logit vectors."""
    return total_variation(S.process(z_a, temperature, top_p), S.process(z_b, temperature, top_p))


def tv_by_depth(zs: Dict[Tuple[int, int], np.ndarray], positions: Sequence[int],
                depths: Sequence[int], R: int, temperature: float,
                top_p: float) -> Dict[int, np.ndarray]:
    """Per-position TV(p_r, p_R) for each depth r, from readout logits keyed
    (position, depth) (e.g. decode.prefill(..., keep_logits=True) with every
    depth as a readout depth)."""
    return {r: np.array([readout_tv(zs[(t, r)], zs[(t, R)], temperature, top_p)
                         for t in positions]) for r in depths}


def fit_envelope(depths: Sequence[int], mean_tv: Sequence[float]) -> Tuple[float, float]:
    """Eq. 7's envelope beta r^-alpha through per-depth mean TVs (readings in
    the module docstring).  Returns (alpha, beta)."""
    r = np.asarray(depths, np.float64)
    m = np.asarray(mean_tv, np.float64)
    use = m > 0
    if use.sum() < 2:
        raise ValueError("need two depths with non-zero mean TV")
    x, y = np.log(r[use]), np.log(m[use])
    slope = float(((x - x.mean()) * (y - y.mean())).sum() / ((x - x.mean()) ** 2).sum())
    alpha = -slope
    beta = float(np.max(m[use] * r[use] ** alpha))
    return alpha, beta


def feasible_pairs(R: int) -> List[Tuple[int, int]]:
    """Integer depth pairs the page's implementation accepts: 1 <= d1 < d2 < R,
    d2 and R multiples of d1."""
    return [(d1, d2) for d1 in range(1, R) if R % d1 == 0
            for d2 in range(2 * d1, R, d1)]


def rank_pairs(alpha: float, beta: float, R: int) -> List[Tuple[int, int]]:
    """Feasible pairs in ascending order of Eq. 11's bound."""
    return sorted(feasible_pairs(R), key=lambda p: (cost_bound(p[0], p[1], R, alpha, beta), p))
