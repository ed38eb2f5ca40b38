"""Second-proposal ablations and mechanism statistics on one configuration.

Runs the same prompt and sampling settings (T = 1 with the configuration's
top-p) in four modes and reports, per mode, what the LoopSpec page tabulates
for its trained models: throughput and speedup over full-depth AR (Table 3),
gamma (R loop passes per token under AR over the depth each committed token was
drafted at) and committed tokens per step, the effective batch -- active rows per shared-block
pass, as a histogram with mean and peak (Fig. 5) --, how often the gate opens
(Table 6) and where committed tokens come from (first proposal, second
proposal, full-depth fallback; Fig. 6).

Modes (section 3.4 of the page): gated (the method: the residual second
proposal opens only when the deeper readout's confidence in the first drops),
ungated (the residual second proposal always), masked (non-residual: a draft
from p_d2 with the first candidate removed and renormalised), single (no
second proposal).

Usage: python -m looped_transformer_self_b200.ablations [model] [tokens]
"""
from __future__ import annotations

import json
import sys
import time

import numpy as np
import torch

import synthetic as syn

from .binding import Decoder

MODES = [("gated", 0, True), ("ungated", 1, True), ("masked", 2, True), ("single", 0, False)]


def _timed(g, n, ar=False):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    toks, st = g.generate(n, ar=ar)
    torch.cuda.synchronize()
    return toks, st, time.perf_counter() - t0


def run(model: str = "ouro14", n: int = 256, max_branches: int = 16, device: str = "cuda"):
    cfg = syn.MODELS[model]
    base = syn.DECODES[f"{model}_sample"].replace(max_new=n)
    prompt = syn.prompt_for(model)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    weights = {k: torch.from_numpy(a).to(device=device, dtype=dt) for k, a in syn.iter_weights(cfg)}
    out = []
    ar_s = None
    for name, mode, two in MODES:
        dec = base if two else base.replace(d2=0)
        g = Decoder(cfg, dec, None, max_branches=max_branches, max_ctx=len(prompt) + n + 16,
                    trace_steps=4 * n + 16, second_mode=mode, device=device)
        g.weights = weights
        g.bind_weights()
        if ar_s is None:
            g.prefill(prompt)
            g.generate(min(n, 32), ar=True)  # warm-up (graph capture)
            g.prefill(prompt)
            _, _, ar_s = _timed(g, n, ar=True)
        g.prefill(prompt)
        g.generate(min(n, 32))  # warm-up
        g.prefill(prompt)
        _, st, sec = _timed(g, n)
        rows = np.array([len(step) for step in g.read_trace(st["steps"])], dtype=np.int64)
        hist = np.bincount(rows, minlength=int(rows.max()) + 1).tolist()
        commits = st["n_first"] + st["n_second"] + st["n_fallback"]
        out.append({
            "mode": name, "tokens": n, "tok_s": n / sec, "ar_tok_s": n / ar_s,
            "speedup_vs_ar": ar_s / sec, "steps": st["steps"], "tokens_per_step": n / st["steps"],
            # loop passes saved: R per token under AR over the depth each token was drafted at
            "gamma": commits * cfg.R / max(st["n_first"] * dec.d1 + st["n_second"] * dec.d2 +
                                           st["n_fallback"] * cfg.R, 1),
            "rows_mean": float(rows.mean()), "rows_peak": int(rows.max()), "rows_hist": hist,
            "gate_checks": st["gate_checks"], "gate_opens": st["gate_opens"],
            "gate_open_rate": st["gate_opens"] / max(st["gate_checks"], 1),
            "src_first": st["n_first"] / max(commits, 1), "src_second": st["n_second"] / max(commits, 1),
            "src_fallback": st["n_fallback"] / max(commits, 1),
        })
        g.close()
        print(json.dumps(out[-1]), flush=True)
    return out


if __name__ == "__main__":
    m = sys.argv[1] if len(sys.argv) > 1 else "ouro14"
    k = int(sys.argv[2]) if len(sys.argv) > 2 else 256
    run(m, k)
