"""Calibrate a random-init looped LM's residual scale and LM-head gain.

The pages evaluate trained checkpoints whose early-loop readouts already agree
with full depth most of the time (LoopSpec page, section 3.1, Fig. 3: top-1
agreement with the final depth).  A random-init model has no such structure,
so two init knobs stand in for training:
  * head gain g (LM head ~ N(0, g^2/d)): set so that the median full-depth
    top-1 probability over the prompt is about 0.3 (readouts are neither flat
    nor one-hot);
  * residual scale s of the shared-block layers: set so that the top-1
    agreement between the first proposal depth and full depth over the prompt
    (teacher-forced prefill readouts) hits the target.
Both are found by bisection on GPU prefill readouts through the C ABI.

Usage: python -m looped_transformer_self_b200.tune ouro14
"""
from __future__ import annotations

import json
import sys

import numpy as np
import torch

import synthetic as syn

from .binding import Decoder


def _head_index(cfg):
    return [n for n, *_ in syn.tensor_specs(cfg)].index("head")


def measure(cfg, dec, prompt, weights_dev, device="cuda"):
    """(agreement of depth d1 with R, median top-1 probability at R)."""
    g = Decoder(cfg, dec, None, max_branches=16, max_ctx=len(prompt) + 8, device=device)
    g.weights = weights_dev
    g.bind_weights()
    _, am, lg = g.prefill(prompt, argmax=True, logits=True)
    tags = sorted({r for r in (dec.d1, dec.d2, cfg.R) if r > 0})
    agree = float(np.mean(am[:, tags.index(dec.d1)] == am[:, tags.index(cfg.R)]))
    zR = lg[:, tags.index(cfg.R)].double()
    top1 = float(torch.softmax(zR, dim=-1).max(dim=-1).values.median())
    g.close()
    return agree, top1


def tune(model: str, target_top1: float = 0.3, iters: int = 10, device="cuda", tol: float = 0.005):
    cfg = syn.MODELS[model]
    dec = syn.DECODES[f"{model}_greedy"]
    d1, target = syn.AGREEMENT_TARGET[model]
    assert d1 == dec.d1
    prompt = syn.prompt_for(model)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    w = {n: torch.from_numpy(a).to(device=device, dtype=dt) for n, a in syn.iter_weights(cfg)}
    hi = _head_index(cfg)
    log = []

    def with_gain(gain):
        c = cfg.replace(head_gain=gain)
        w["head"] = torch.from_numpy(syn.make_tensor(c, hi)[1]).to(device=device, dtype=dt)
        return c

    # head gain: median top-1 probability increases with g
    lo_g, hi_g = 0.5, 12.0
    for _ in range(iters):
        mid = 0.5 * (lo_g + hi_g)
        a, t1 = measure(with_gain(mid), dec, prompt, w, device)
        log.append(("gain", mid, cfg.resid_scale, a, t1))
        if t1 < target_top1:
            lo_g = mid
        else:
            hi_g = mid
    gain = round(0.5 * (lo_g + hi_g), 3)
    c = with_gain(gain)
    # residual scale: agreement decreases as s grows.  The useful scales span
    # orders of magnitude (~0.005 for Huginn-3.5B, ~0.014 for Ouro-1.4B), so
    # the bisection runs on log s; it stops once the agreement is within tol of
    # the target, and the evaluated scale closest to the target wins.
    lo_s, hi_s = np.log(1e-4), np.log(2.0)
    best = None
    for _ in range(2 * iters):
        mid = float(np.exp(0.5 * (lo_s + hi_s)))
        mid = float(f"{mid:.4g}")
        a, t1 = measure(c.replace(resid_scale=mid), dec, prompt, w, device)
        log.append(("scale", gain, mid, a, t1))
        if best is None or abs(a - target) < abs(best[1] - target):
            best = (mid, a, t1)
        if abs(a - target) <= tol:
            break
        if a > target:
            lo_s = np.log(mid)
        else:
            hi_s = np.log(mid)
    s, a, t1 = best
    return {"model": model, "head_gain": gain, "resid_scale": s, "agreement": a,
            "median_top1": t1, "target_agreement": target, "log": log}


if __name__ == "__main__":
    out = [tune(m) for m in (sys.argv[1:] or ["ouro14"])]
    print(json.dumps(out, indent=1))
