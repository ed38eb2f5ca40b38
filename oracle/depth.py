"""Depth selection of the LoopSpec page, section 2.4 (test infrastructure only).

Eq. 7 bounds the mean total variation between the depth-r readout and the
target by a power law beta * r^-alpha; Eq. 11 bounds the expected serial loop
steps per committed token by d1 + beta d1^-alpha d2 + 2 beta d2^-alpha R; its
stationary point is Eq. 8:
    D = alpha^2 + alpha + 1,
    d1* = (alpha beta)^((alpha+1)/D) (2 alpha R)^(1/D),
    d2* = (alpha beta)^(alpha/D) (2 alpha R)^((alpha+1)/D).
"""
from __future__ import annotations

from typing import Tuple


def cost_bound(d1: float, d2: float, R: float, alpha: float, beta: float) -> float:
    """Eq. 11 right-hand side."""
    return d1 + beta * d1 ** -alpha * d2 + 2.0 * beta * d2 ** -alpha * R


def optimal_depths(alpha: float, beta: float, R: float) -> Tuple[float, float]:
    """Eq. 8: continuous stationary point of the Eq. 11 bound."""
    D = alpha * alpha + alpha + 1.0
    d1 = (alpha * beta) ** ((alpha + 1.0) / D) * (2.0 * alpha * R) ** (1.0 / D)
    d2 = (alpha * beta) ** (alpha / D) * (2.0 * alpha * R) ** ((alpha + 1.0) / D)
    return d1, d2
