"""Kernel sweep of one mixed-depth shared-block step (Ouro-shaped, bf16).

M = 1, 2, 4, 8, 16, 32, 64 active rows; each row at an independent depth 1..4
with its own KV length drawn uniformly from 256..8192 (synthetic.sweep_rows),
its own randomly permuted (or, --order seq, ascending) cache slots, caches and hidden states N(0, 1).  One
pass = all 24 shared layers over the M rows (lt_block_pass), captured as a
CUDA graph and replayed; reported: median pass time, algorithmic bytes
(shared-block weights + every row's K/V reads and writes) and GB/s against the
measured HBM copy bandwidth.

Usage: python -m looped_transformer_self_b200.sweep [M ...] [--layers N] [--iters K] [--order perm|seq]
"""
from __future__ import annotations

import json
import os
import statistics
import sys

import numpy as np
import torch

import synthetic as syn

from .binding import Decoder

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run(Ms=(1, 2, 4, 8, 16, 32, 64), iters=50, device="cuda", layers=None, order="perm"):
    cfg = syn.MODELS["sweep"]
    if layers:  # fewer shared layers: a small case of the same kernels (profilers)
        cfg = cfg.replace(n_core=layers)
    d = cfg.d_model
    try:
        hbm = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["hbm_gbs"]
    except Exception:
        hbm = 6650.0
    dt = torch.bfloat16
    weights = {n: torch.from_numpy(a).to(device=device, dtype=dt) for n, a in syn.iter_weights(cfg)}
    wbytes = 2.0 * cfg.n_core * (4 * d * d + 3 * d * cfg.ffn)
    out = []
    for M in Ms:
        C = next(c for c in (8, 16, 32, 64) if c >= M)
        depth, lens = syn.sweep_rows(M, cfg.R)
        rng = np.random.default_rng(3)
        nxt, lists, offs = {}, [], []
        for r, l in zip(depth.tolist(), lens.tolist()):
            start = nxt.get(r, 0)
            nxt[r] = start + l + 1
            offs.append(sum(len(x) for x in lists))
            sl = np.arange(start, start + l + 1)
            lists.append((rng.permutation(sl) if order == "perm" else sl).astype(np.int32))
        S = max(nxt.values())
        g = Decoder(cfg, syn.DecodeConfig(1, 2, 0.0, 1.0, 2, 1), None, max_branches=C,
                    max_ctx=max(S, 8200), device=device)
        g.weights = weights
        g.bind_weights()
        pool, _ = g.kv_pool()
        gen = torch.Generator(device=device).manual_seed(3)
        for p in range(pool.shape[0]):
            pool[p].normal_(generator=gen)
        hid = torch.randn(M, d, generator=gen, device=device)
        ms = g.block_pass(depth, lens, torch.from_numpy(np.concatenate(lists)).to(device),
                          np.array(offs, np.int32), hid, iters=iters, timed=True)
        med = statistics.median(ms[3:]) if len(ms) > 4 else statistics.median(ms)
        kv = float(sum(cfg.n_core * (l + 1) * 2 * d * 2 for l in lens.tolist()))
        gbs = (wbytes + kv) / (med / 1e3) / 1e9
        row = {"M": M, "C": C, "median_ms": med, "weight_bytes": wbytes, "kv_bytes": kv,
               "gbs": gbs, "frac_of_measured_hbm": gbs / hbm,
               "mean_len": float(np.mean(lens)), "depths": depth.tolist()}
        out.append(row)
        print(json.dumps(row), flush=True)
        g.close()
        del pool, hid
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    import argparse
    ap = argparse.ArgumentParser()
    ap.add_argument("M", type=int, nargs="*", default=[1, 2, 4, 8, 16, 32, 64])
    ap.add_argument("--layers", type=int, default=None, help="shared layers (default 24)")
    ap.add_argument("--iters", type=int, default=50, help="graph replays per M")
    ap.add_argument("--order", choices=("perm", "seq"), default="perm",
                    help="slot order of each row's list: permuted (default) or ascending")
    a = ap.parse_args()
    run(tuple(a.M), iters=a.iters, layers=a.layers, order=a.order)
