"""Decode steps inside a CUDA profiler range, for kernel profilers.

Builds a decoder for one of the synthetic model configurations, prefills its
prompt, decodes ``--warm`` tokens (graphs captured, caches filled), then runs
``--window`` single decode steps between cudaProfilerStart and
cudaProfilerStop.  Run it under ``ncu --profile-from-start off`` to capture
only those steps' kernel launches, e.g.

    ncu --metrics gpu__time_duration.sum --clock-control none \\
        --profile-from-start off --csv --log-file launches.csv \\
        python -m looped_transformer_self_b200.profile_step --model ouro14 --window 8
"""
import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402
from looped_transformer_self_b200.binding import Decoder  # noqa: E402


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--model", default="ouro14")
    ap.add_argument("--warm", type=int, default=96, help="tokens decoded before the window")
    ap.add_argument("--window", type=int, default=8, help="decode steps profiled")
    ap.add_argument("--sampled", action="store_true", help="temperature sampling instead of greedy")
    args = ap.parse_args()
    cfg = syn.MODELS[args.model]
    dec = syn.DECODES[f"{args.model}_{'sample' if args.sampled else 'greedy'}"]
    n = args.warm + args.window + 8
    dec = dec.replace(max_new=n)
    prompt = syn.prompt_for(args.model)
    g = Decoder(cfg, dec, syn.make_weights(cfg), max_branches=16, max_ctx=len(prompt) + n + 16)
    g.prefill(prompt)
    g.generate(args.warm)
    torch.cuda.synchronize()
    torch.cuda.profiler.start()
    for _ in range(args.window):
        g.step()
    torch.cuda.synchronize()
    torch.cuda.profiler.stop()
    g.close()
    print(f"profiled {args.window} decode steps of {args.model}")


if __name__ == "__main__":
    main()
