"""Proposal depths from measured readout divergence.

LoopSpec page, section 2.4: the mean total variation between the depth-r
readout and the full-depth target is bounded by a power law beta r^-alpha
(Eq. 7); with it, the expected serial loop steps per committed token are
bounded by d1 + beta d1^-alpha d2 + 2 beta d2^-alpha R (Eq. 11), whose
stationary point is Eq. 8.  Section 3.1 (Fig. 3 right) measures the TV at
T = 1, top-p 0.7, averaged over positions, for ten depths, and draws the
power law as an upper envelope.  The page takes Eq. 8 as the start of a
search: the implementation needs integers 1 <= d1 < d2 < R with d2 and R
multiples of d1, and the final choice is the best measured wall clock.

This module does those steps for one model:
  1. readouts at depth r and R of every prompt position (one prefill per r
     with d1 = r) and their TV per position (lt_readout_tv, on the device);
  2. the envelope: alpha by least squares on (ln r, ln mean TV) over depths
     with non-zero mean, beta the smallest value with beta r^-alpha >= every
     mean;
  3. Eq. 8's continuous (d1*, d2*) and the feasible integer pairs ranked by
     Eq. 11's bound;
  4. a wall-clock sweep of the best-ranked pairs (speculative decoding at the
     same T and top-p) against full-depth AR.

Usage: python -m looped_transformer_self_b200.depth_select [model] [tokens] [candidates]
"""
from __future__ import annotations

import json
import math
import sys
import time
from typing import Dict, List, Sequence, Tuple

import numpy as np

# ---------------------------------------------------------------------------
# host logic (no GPU needed)
# ---------------------------------------------------------------------------


def default_depths(R: int, count: int = 10) -> List[int]:
    """The first `count` depths below R (Fig. 3 right measures ten)."""
    return list(range(1, min(count, R - 1) + 1))


def envelope(depths: Sequence[int], mean_tv: Sequence[float]) -> Tuple[float, float]:
    """(alpha, beta) of the power-law upper envelope of Eq. 7."""
    pts = [(math.log(r), math.log(m), r, m) for r, m in zip(depths, mean_tv) if m > 0]
    if len(pts) < 2:
        raise ValueError("need two depths with non-zero mean TV")
    n = len(pts)
    xm = sum(p[0] for p in pts) / n
    ym = sum(p[1] for p in pts) / n
    sxx = sum((p[0] - xm) ** 2 for p in pts)
    sxy = sum((p[0] - xm) * (p[1] - ym) for p in pts)
    alpha = -sxy / sxx
    beta = max(m * r ** alpha for _, _, r, m in pts)
    return alpha, beta


def eq8(alpha: float, beta: float, R: int) -> Tuple[float, float]:
    """Continuous optimal depths (Eq. 8)."""
    den = alpha * alpha + alpha + 1.0
    ab, ar2 = alpha * beta, 2.0 * alpha * R
    return ab ** ((alpha + 1.0) / den) * ar2 ** (1.0 / den), ab ** (alpha / den) * ar2 ** ((alpha + 1.0) / den)


def loop_step_bound(d1: float, d2: float, R: int, alpha: float, beta: float) -> float:
    """Eq. 11: expected serial loop steps per committed token, upper bound."""
    return d1 + beta * d2 / d1 ** alpha + 2.0 * beta * R / d2 ** alpha


def candidate_pairs(R: int) -> List[Tuple[int, int]]:
    """Integer pairs with 1 <= d1 < d2 < R and d2, R multiples of d1."""
    out = []
    for d1 in range(1, R):
        if R % d1:
            continue
        d2 = 2 * d1
        while d2 < R:
            out.append((d1, d2))
            d2 += d1
    return out


def ranked_pairs(alpha: float, beta: float, R: int) -> List[Tuple[int, int]]:
    return sorted(candidate_pairs(R),
                  key=lambda p: (loop_step_bound(p[0], p[1], R, alpha, beta), p))


# ---------------------------------------------------------------------------
# measurement (GPU)
# ---------------------------------------------------------------------------


def measure_tv(cfg, dec, weights, prompt, depths, temperature=1.0, top_p=0.7,
               max_branches=16, device="cuda") -> Dict[int, np.ndarray]:
    """Per-position TV(p_r, p_R) of the prompt's positions for each r in depths.
    `weights`: dict of device tensors (shared by the handles) or host arrays."""
    import torch

    from .binding import Decoder, readout_tv
    out = {}
    for r in depths:
        g = Decoder(cfg, dec.replace(d1=r, d2=0), None, max_branches=max_branches,
                    max_ctx=len(prompt) + 16, device=device)
        if isinstance(weights, dict) and all(isinstance(v, torch.Tensor) for v in weights.values()):
            g.weights = weights
            g.bind_weights()
        else:
            g.load(weights)
        _, _, lg = g.prefill(prompt, logits=True)  # [n][2][V]: depth r, then R
        tv = readout_tv(lg[:, 0, :], lg[:, 1, :], temperature, top_p, stream=g.stream)
        g.stream.synchronize()
        out[r] = tv.cpu().numpy().astype(np.float64)
        del lg
        g.close()
    return out


def sweep(cfg, dec, weights, prompt, pairs, n, want=None, device="cuda"):
    """Decode throughput (tokens/s, device clock) of speculative decoding at
    (d1, d2) pairs taken in order, and of full-depth AR (one row: the smallest
    branch table).  Pairs whose branch tree outgrows the largest table (64
    rows) are reported with their error; with `want`, the sweep stops once that
    many pairs were measured (or 6 * want were tried)."""
    import torch

    from .binding import Decoder, LoopedSpecError

    def timed(g, ar):
        g.prefill(prompt)
        g.generate(min(n, 16), ar=ar)  # graph capture, caches warm
        g.prefill(prompt)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(g.stream)
        _, st = g.generate(n, ar=ar)
        e1.record(g.stream)
        torch.cuda.synchronize()
        return n / (e0.elapsed_time(e1) / 1e3), st

    def handle(d1, d2, C):
        g = Decoder(cfg, dec.replace(d1=d1, d2=d2, max_new=n), None, max_branches=C,
                    max_ctx=len(prompt) + n + 32, device=device)
        g.weights = weights
        g.bind_weights()
        return g

    g = handle(*pairs[0], 8)
    ar_tok_s, _ = timed(g, True)
    g.close()
    res = {}
    for d1, d2 in pairs:
        if want is not None and (sum(1 for v in res.values() if v["tok_s"]) >= want or
                                 len(res) >= 6 * want):
            break
        # rows in flight grow like R / d1 (a new branch every d1 loop steps, each
        # alive for R); start from that estimate and grow the table on overflow
        est = rows_estimate(cfg.R, d1, d2)
        sizes = [c for c in (8, 16, 32, 64) if c >= min(est, 64)]
        for C in sizes:
            g = handle(d1, d2, C)
            try:
                tok_s, st = timed(g, False)
            except LoopedSpecError as e:
                g.close()
                if e.code == -3 and C < sizes[-1]:  # LT_ERR_CAPACITY: next table size
                    continue
                res[(d1, d2)] = {"tok_s": None, "error": str(e), "max_branches": C}
                break
            res[(d1, d2)] = {"tok_s": tok_s, "steps": st["steps"], "max_branches": C,
                             "rows_max": st["rows_max"], "n_first": st["n_first"],
                             "n_second": st["n_second"], "n_fallback": st["n_fallback"]}
            g.close()
            break
    return ar_tok_s, res


def rows_estimate(R: int, d1: int, d2: int) -> int:
    """Rows in flight with proposals every d1 loop steps: about R / d1 branches
    on the committed chain plus (R - d2) / d1 second-proposal branches."""
    return -(-R // d1) + max(R - d2, 0) // d1 + 1


def run(model="ouro14", n=256, candidates=6, temperature=1.0, top_p=0.7, tv_positions=256,
        device="cuda"):
    import torch

    import synthetic as syn
    cfg = syn.MODELS[model]
    dec = syn.DECODES[f"{model}_sample"].replace(temperature=temperature, top_p=top_p)
    prompt = syn.prompt_for(model)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    weights = {k: torch.from_numpy(a).to(device=device, dtype=dt) for k, a in syn.iter_weights(cfg)}
    depths = default_depths(cfg.R)
    t0 = time.time()
    tv = measure_tv(cfg, dec, weights, prompt[:tv_positions], depths, temperature, top_p,
                    device=device)
    means = [float(tv[r].mean()) for r in depths]
    alpha, beta = envelope(depths, means)
    c1, c2 = eq8(alpha, beta, cfg.R)
    ranked = ranked_pairs(alpha, beta, cfg.R)
    ar, res = sweep(cfg, dec, weights, prompt, ranked, n, want=candidates, device=device)
    # the configured pair and the page's measured choice for R = 32, for comparison
    extra = [p for p in [(dec.d1, dec.d2), (2, 8)] if p in candidate_pairs(cfg.R) and p not in res]
    if extra:
        res.update(sweep(cfg, dec, weights, prompt, extra, n, device=device)[1])
    pick = list(res)
    ok = [p for p in pick if res[p]["tok_s"]]
    best = max(ok, key=lambda p: res[p]["tok_s"])
    first_ok = next(p for p in ranked if p in ok)
    return {
        "model": model, "R": cfg.R, "T": temperature, "top_p": top_p,
        "tv_positions": len(prompt[:tv_positions]), "depths": depths, "mean_tv": means,
        "alpha": alpha, "beta": beta, "eq8": [c1, c2],
        "ranked": [[d1, d2, loop_step_bound(d1, d2, cfg.R, alpha, beta)] for d1, d2 in pick],
        "tokens": n, "ar_tok_s": ar,
        "sweep": [dict(d1=d1, d2=d2, speedup_vs_ar=(res[(d1, d2)]["tok_s"] or 0.0) / ar,
                       **res[(d1, d2)]) for d1, d2 in pick],
        "formula_pick": list(ranked[0]), "formula_pick_measured": list(first_ok),
        "measured_best": list(best),
        "formula_pick_vs_best": res[first_ok]["tok_s"] / res[best]["tok_s"],
        "seconds": time.time() - t0,
    }


if __name__ == "__main__":
    m = sys.argv[1] if len(sys.argv) > 1 else "ouro14"
    k = int(sys.argv[2]) if len(sys.argv) > 2 else 256
    c = int(sys.argv[3]) if len(sys.argv) > 3 else 6
    print(json.dumps(run(m, k, c)))
