"""Decode benchmark: pipelined self-speculative decoding of a looped LM on B200.

Default workload (the pages' single-request decode setting, LoopSpec page
section 3.1, on the largest configuration that fits one GPU): a Huginn/Raven-
3.5B-shaped looped LM (bf16, random init with the residual scale tuned for
depth-8 vs depth-32 top-1 agreement ~0.7; prelude 2 layers, core block 4
layers looped R = 32, coda 2 layers; d 5280, 55 x 96 heads, SwiGLU 17920,
vocab 65536), a 256-token Zipf(1.1) prompt, 512 decoded tokens, proposal
readouts at depths 8 and 16.  `--model ouro14 | ouro26 | tiny` selects the
other workloads.

One bench step = prefill (untimed: the pages time the decode phase only) +
one greedy pipelined speculative decode of the workload's tokens through the
C ABI, timed with CUDA events on the decoder's stream.  value = decoded
tokens / s summed over ranks (replicas: one independent request per GPU, no
collective on the data path).  The shared block's weights exceed the 126 MB
L2, so no flush is needed between steps.

`--impl reference` times the CPU oracle (the plain fp64 implementation the
GPU path is checked against) on the host cores on a bounded sample of the
same workload.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402


def _peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return None


class Clocks:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index, self.samples, self.stop = index, [], threading.Event()

    def _run(self):
        while not self.stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                      "--format=csv,noheader,nounits"], capture_output=True,
                                     text=True, timeout=5).stdout.strip()
                if out:
                    self.samples.append([x.strip() for x in out.split(",")])
            except Exception:
                pass
            self.stop.wait(0.2)

    def __enter__(self):
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def __exit__(self, *a):
        self.stop.set()
        self.t.join(timeout=10)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for s in self.samples for k in range(4)
                          if len(s) > 4 + k and s[4 + k].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.samples)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 0, 1
    import datetime
    import torch.distributed as dist
    rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
    backend = "nccl" if os.environ.get("BENCH_BACKEND", "nccl") == "nccl" else "gloo"
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    return rank, local, ws


def _max_over_ranks(x, ws, device):
    if ws <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------------------
# CPU oracle baseline (also the --impl reference arm)
# ---------------------------------------------------------------------------

# bounded oracle samples per workload (prompt tokens kept, decode tokens timed
# per sample): about 10-30 s of fp64 host work for the CPU baseline; the
# reference arm times one sample per step
ORACLE_SAMPLE = {"tiny": (32, 64), "ouro14": (8, 24), "huginn35": (2, 2), "ouro26": (8, 16)}
REFERENCE_SAMPLE = {"tiny": (32, 16), "ouro14": (8, 4), "huginn35": (2, 1), "ouro26": (8, 4)}


class OracleSample:
    """The CPU oracle on a bounded sample of a workload: the prompt truncated
    to n_prompt tokens is prefilled once (untimed, as the metric excludes
    prefill), its caches are kept, and each timed sample restores them and
    runs the oracle's pipelined speculative decoder for n_tokens tokens."""

    def __init__(self, cfg, dec, prompt, weights, n_prompt, n_tokens, copy=None):
        from oracle import decode as D
        from oracle.model import LoopedModel
        self.D, self.cfg, self.dec = D, cfg, dec
        self.n_prompt, self.n_tokens = n_prompt, n_tokens
        self.prompt = list(prompt[:n_prompt])
        self.n_slots = n_prompt + n_tokens + 24
        self.cp = None if copy is None else D.CopyConfig(
            tau=copy.tau, k=copy.k, max_len=copy.max_len, match_cap=copy.match_cap, table=32,
            reserve=copy.reserve)
        t0 = time.perf_counter()
        self.model = LoopedModel(cfg, weights, self.n_slots)
        self.rows = D.OracleRows(self.model)
        tags = D.readout_depths(cfg.R, dec.d1, dec.d2)
        zs = D.prefill(self.rows, self.prompt, cfg.R, tags)
        self.first = D.first_token(zs[(n_prompt - 1, cfg.R)], n_prompt, dec.temperature,
                                   dec.top_p, dec.seed)
        self.snap = {k: (K.copy(), V.copy()) for k, (K, V) in self.model.caches.items()}
        self.prefill_s = time.perf_counter() - t0

    def run(self):
        """One timed sample: decode seconds."""
        for k, (K, V) in self.snap.items():
            Kc, Vc = self.model.cache(*k)
            Kc[:] = K
            Vc[:] = V
        for k in list(self.model.caches):
            if k not in self.snap:
                del self.model.caches[k]
        D, cfg, dec = self.D, self.cfg, self.dec
        t1 = time.perf_counter()
        D.SpecDecoder(self.rows, self.prompt, cfg.R, dec.d1, dec.d2, self.n_tokens,
                      dec.temperature, dec.top_p, dec.seed, self.n_slots, keep_trace=False,
                      skip_prefill=True, first=self.first, copy=self.cp).run()
        return time.perf_counter() - t1

    def describe(self, decode_s):
        return (f"{self.cfg.name}: prompt truncated to {self.n_prompt} tokens (prefilled once, "
                f"{self.prefill_s:.1f} s, untimed), {self.n_tokens} greedy pipelined speculative "
                f"decode tokens per sample (d1={self.dec.d1}, d2={self.dec.d2}), decode "
                f"{decode_s:.1f} s timed, fp64 on {os.cpu_count()} host threads")


def oracle_baseline(cfg, dec, prompt, weights, model, copy=None):
    n_prompt, n_tokens = ORACLE_SAMPLE[model]
    o = OracleSample(cfg, dec, prompt, weights, n_prompt, n_tokens, copy)
    t = o.run()
    return {"value": n_tokens / t, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": o.describe(t)}


def run_reference(args):
    import synthetic as syn
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg = syn.MODELS[args.model]
    dec = syn.DECODES[f"{args.model}_greedy"]
    prompt = syn.prompt_for(args.model)
    n_prompt, n_tokens = REFERENCE_SAMPLE[args.model]
    o = OracleSample(cfg, dec, prompt, syn.make_weights(cfg), n_prompt, n_tokens)
    for _ in range(args.warmup):
        o.run()
    times = [o.run() for _ in range(max(1, args.steps))]
    v = n_tokens * len(times) / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOADS.get(args.model, args.model),
                       "l2": "weights larger than L2"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(),
                             "kind": "oracle", "sample": o.describe(sum(times))},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


METRIC = "decoded tokens/s at batch 1 (greedy, T=1) + step HBM GB/s vs 8 TB/s"
WORKLOADS = {
    "huginn35": ("huginn35: Huginn/Raven-3.5B-shaped looped LM (bf16, prelude 2 + core 4 x R=32 "
                 "+ coda 2 layers, d5280, 55x96, ffn17920, V65536), 256-token Zipf(1.1) prompt, "
                 "512 decode tokens, proposals at depths 8 and 16, batch 1"),
    "ouro14": ("ouro14: Ouro-1.4B-shaped looped LM (bf16, 24 shared layers x R=4, d2048, 16x128, "
               "ffn5632, V49152), 512-token Zipf(1.1) prompt, 1024 decode tokens, proposals at "
               "depths 1 and 2, batch 1"),
    "ouro26": ("ouro26: Ouro-2.6B-shaped looped LM (bf16, 48 shared layers x R=4, d2048, 16x128, "
               "ffn5632, V49152), 4096-token Zipf(1.1) prompt with 40% copied 16-64-token spans, "
               "2048 decode tokens, proposals at depths 1 and 2, batch 1"),
    "tiny": ("tiny: looped LM (fp32, prelude 1 + shared 2 x R=4 + coda 1, d128, 4x32, ffn384, "
             "V512), 32-token uniform prompt, 64 decode tokens, proposals at depths 2 and 3"),
}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def gemm_traffic(model, bytes_per_launch, path=None):
    """DRAM traffic per launch of the dominant kernel, from the committed ncu
    capture (profiles/gemm_traffic.json), and a note saying where it came from.
    Reported only while the GEMM sources hash to the captured ones and the
    capture covers this model's shapes: the capture's traffic / algorithmic
    ratio over the four shared-block GEMM shapes, applied to this run's
    algorithmic bytes per launch.  (None, reason) otherwise."""
    path = path or os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(path):
        return None, "no capture"
    from looped_transformer_self_b200.gemm_traffic import source_hash
    cap = json.load(open(path))
    if cap.get("source_sha256") != source_hash():
        return None, "GEMM sources changed since the capture"
    if cap.get("model") != model:
        return None, f"the capture covers the {cap.get('model')} shapes"
    ratio = cap["traffic_per_launch"] / cap["algorithmic_per_launch"]
    return ratio * bytes_per_launch, (
        "ncu dram bytes read + written of the four shared-block GEMM shapes "
        f"(profiles/gemm_traffic.json, ratio to algorithmic {ratio:.4f}); "
        "the GEMM sources match the capture")


def run_ours(args):
    import torch
    import synthetic as syn
    from looped_transformer_self_b200.binding import CopyConfig, Decoder, lib, ProfileC, InfoC
    from looped_transformer_self_b200 import copyloop
    import ctypes

    rank, local, ws = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    cfg = syn.MODELS[args.model]
    n_new = args.n_new or syn.DECODES[f"{args.model}_greedy"].max_new
    dec_g = syn.DECODES[f"{args.model}_greedy"].replace(max_new=n_new, seed=2 + rank)
    prompt = syn.prompt_for(args.model, seed=1 + rank)
    P = len(prompt)
    t_w = time.time()
    weights = syn.make_weights(cfg)
    C = 16 if cfg.R <= 32 else 32
    g = Decoder(cfg, dec_g, weights, max_branches=C, max_ctx=P + 1 + n_new + 8,
                trace_steps=0, device=dev)
    t_w = time.time() - t_w

    # agreement of the depth-d1 readout with full depth over the prompt
    _, am, _ = g.prefill(prompt, argmax=True)
    tags = sorted({r for r in (dec_g.d1, dec_g.d2, cfg.R) if r > 0})
    agree = float(np.mean(am[:, tags.index(dec_g.d1)] == am[:, tags.index(cfg.R)]))

    # context-copy proposals (the Ouro-2.6B workload): tau calibrated on the
    # prompt; the LoopSpec-only handle g stays for comparison
    copy_on = args.copy == "on" or (args.copy == "auto" and args.model == "ouro26")
    copy_info, g_plain = None, None
    cc = None
    if copy_on:
        # calibration text: another prompt of the same recipe (not the timed
        # one), 1024 tokens, and 512 tokens the decoder continues it with
        cal_prompt = syn.prompt_for(args.model, seed=1001 + rank)[:1024]
        cal = copyloop.calibrate(g, cal_prompt, warm=512)
        slack = -(-cfg.R // dec_g.d1) + max(cfg.R - dec_g.d2, 0) // dec_g.d1 + 1
        cc = CopyConfig(tau=cal["tau"], reserve=slack)
        copy_info = {"calibration": cal, "k": cc.k, "max_len": cc.max_len,
                     "match_cap": cc.match_cap, "reserve": cc.reserve, "max_branches": 32,
                     "copied_prompt_fraction": syn.copy_prompt(P, cfg.vocab, 1 + rank)[1]}
        if cal["admitted"] == 0:
            # the calibration admits no copy proposal: decode without them
            copy_info["decision"] = "off (no prompt proposal is more likely accepted than not)"
            copy_on, cc = False, None
        else:
            copy_info["decision"] = "on"
            g_plain = g
            g = Decoder(cfg, dec_g, None, max_branches=32, max_ctx=P + 1 + n_new + 8,
                        trace_steps=0, device=dev, copy=cc)
            g.weights = g_plain.weights
            g.bind_weights()

    def one_generate(ar=False):
        g.prefill(prompt)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(g.stream)
        toks, st = g.generate(n_new, ar=ar)
        e1.record(g.stream)
        e1.synchronize()
        return e0.elapsed_time(e1), toks, st

    for _ in range(args.warmup):
        one_generate()
    _barrier(ws)
    torch.cuda.synchronize()
    times, stats = [], None
    with Clocks(local) as clk:
        for _ in range(args.steps):
            ms, toks, stats = one_generate()
            times.append(ms)
    torch.cuda.synchronize()
    _barrier(ws)
    total_ms = _max_over_ranks(sum(times), ws, dev)
    value = ws * n_new * args.steps / (total_ms / 1000.0)

    # full-depth AR baseline and sampled decoding (same kernels), one run each
    ar_ms, ar_toks, ar_st = one_generate(ar=True)
    spec_equal_ar = ar_toks == toks
    if g_plain is not None:  # LoopSpec proposals only, same prompt
        g_plain.prefill(prompt)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(g_plain.stream)
        plain_toks, plain_st = g_plain.generate(n_new)
        e1.record(g_plain.stream)
        e1.synchronize()
        copy_info.update(loopspec_only_tokens_per_s=n_new / (e0.elapsed_time(e1) / 1e3),
                         loopspec_only_stats=plain_st,
                         loopspec_only_equals_ar=plain_toks == ar_toks,
                         copy_vs_loopspec_only=(e0.elapsed_time(e1)) / times[-1])
        g_plain.close()
    if copy_info is not None:  # every copy proposal admitted (tau = 0), for context
        g_f = Decoder(cfg, dec_g, None, max_branches=32, max_ctx=P + 1 + n_new + 8, device=dev,
                      copy=CopyConfig(tau=0.0, reserve=copy_info["reserve"]))
        g_f.weights = g.weights
        g_f.bind_weights()
        g_f.prefill(prompt)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(g_f.stream)
        f_toks, f_st = g_f.generate(n_new)
        e1.record(g_f.stream)
        e1.synchronize()
        copy_info.update(forced_tau0_tokens_per_s=n_new / (e0.elapsed_time(e1) / 1e3),
                         forced_tau0_stats=f_st, forced_tau0_equals_ar=f_toks == ar_toks)
        g_f.close()
    g_s = Decoder(cfg, syn.DECODES[f"{args.model}_sample"].replace(max_new=n_new, seed=2 + rank),
                  None, max_branches=32 if copy_on else C, max_ctx=P + 1 + n_new + 8, device=dev,
                  copy=cc if copy_on else None)
    g_s.weights = g.weights
    g_s.bind_weights()
    g_s.prefill(prompt)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(g_s.stream)
    _, st_s = g_s.generate(n_new)
    e1.record(g_s.stream)
    e1.synchronize()
    sample_ms = e0.elapsed_time(e1)

    # per-step breakdown: CUDA events around every GEMM and attention launch of
    # 64 un-graphed decode steps (on the decoder's stream)
    g.prefill(prompt)
    prof = g.profile(64)
    info = g.info()
    # live roofline of the dominant kernel in its graphed regime: one pass's
    # shared-block GEMMs captured alone as a graph (programmatic dependent
    # launch between them, as in the step), replayed with CUDA events around
    # the replays on the decoder's stream (resets the decode state)
    pg = g.profile_gemms(20)

    # end to end through the public API: host prompt in, host tokens out
    t0 = time.perf_counter()
    first, _, _ = g.prefill(prompt)
    toks_e2e, _ = g.generate(n_new)
    torch.cuda.synchronize()
    e2e_s = time.perf_counter() - t0

    peaks = _peaks()
    hbm = peaks["hbm_gbs"] if peaks else 6650.0
    gemm_gbs = pg["bytes"] / (pg["ms"] / 1e3) / 1e9
    gemm_gbs_ungraphed = prof["gemm_core_bytes"] / (prof["gemm_core_ms"] / 1e3) / 1e9
    # algorithmic bytes of an average step (shared-block weights, prelude / coda /
    # LM-head weights on the steps that run them, KV reads and writes), over the
    # graphed step time of the timed decode
    step_bytes = (prof["gemm_core_bytes"] + prof["gemm_other_bytes"] + prof["kv_bytes"]) / max(prof["steps"], 1)
    graphed_ms = times[-1] / stats["steps"]
    step_gbs = step_bytes / (graphed_ms / 1e3) / 1e9
    traffic, traffic_note = gemm_traffic(args.model, pg["bytes"] / pg["launches"])

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu:
        cpu = oracle_baseline(cfg, dec_g, prompt, weights, args.model,
                              copy=cc if copy_on else None)

    if rank == 0:
        n_steps = stats["steps"]
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOADS.get(args.model, args.model),
                       "parallelism": f"replicas x{ws}",
                       "l2": ("no flush: the shared block's weights (%.2f GB per pass) exceed the "
                              "126 MB L2" % (info["weight_bytes_core"] / 1e9)),
                       "resid_scale": cfg.resid_scale, "agreement_d1_vs_R": agree,
                       "max_branches": 32 if copy_on else C, "n_new": n_new, "prompt_len": P},
            "speedup_vs_full_depth_ar": (ar_ms / times[-1]),
            "ar_tokens_per_s": n_new / (ar_ms / 1e3),
            "sampled_tokens_per_s": n_new / (sample_ms / 1e3),
            "spec_greedy_equals_ar_greedy": bool(spec_equal_ar),
            "gamma": _gamma(stats, dec_g.d1, dec_g.d2, cfg.R),
            "gamma_sampled": _gamma(st_s, dec_g.d1, dec_g.d2, cfg.R),
            "decode_stats": stats, "sampled_stats": st_s,
            "step_hbm": {"gbs": step_gbs, "frac_of_measured_hbm": step_gbs / hbm,
                         "frac_of_8_tbs": step_gbs / 8000.0,
                         "bytes_per_step": step_bytes, "ms_per_step_graphed": graphed_ms,
                         "ms_per_step_profiled": prof["step_ms"] / max(prof["steps"], 1),
                         "peak_source": "measured" if peaks else "fallback"},
            "roofline": {"kernel": "k_gemm (tcgen05 weight-streaming GEMM)", "bound": "hbm",
                         "achieved": gemm_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": gemm_gbs / hbm, "traffic": traffic,
                         "traffic_note": traffic_note,
                         "peak_source": ("measured (burst copy, MEASURED_PEAKS.json)" if peaks
                                         else "fallback"),
                         "timing": ("one decode pass's %d shared-block GEMM launches captured "
                                    "alone as a CUDA graph, 20 replays, CUDA events on the "
                                    "decoder's stream: %.3f ms per replay" % (pg["launches"], pg["ms"])),
                         "algorithmic_bytes_per_launch": pg["bytes"] / pg["launches"],
                         "avg_launch_us": 1e3 * pg["ms"] / pg["launches"],
                         "ungraphed_gbs": gemm_gbs_ungraphed},
            "cpu_baseline": cpu,
            "e2e": {"value": n_new / e2e_s, "unit": "tokens/s",
                    "h2d_bytes_per_step": 4 * P, "d2h_bytes_per_step": 4 * (n_new + 1),
                    "includes": "lt_prefill + lt_generate wall time, host buffers"},
            "copy_proposals": copy_info,
            "gpu_launches": info["kernels_per_step"] * n_steps * args.steps,
            "clocks": clk.summary(),
            "profile": prof,
            "weights_gen_s": t_w,
        }
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def _gamma(st, d1, d2, R):
    den = st["n_first"] * d1 + st["n_second"] * d2 + st["n_fallback"] * R
    n = st["n_first"] + st["n_second"] + st["n_fallback"]
    return n * R / den if den else None


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--model", default="huginn35", choices=sorted(WORKLOADS),
                    help="workload (default: the largest single-GPU configuration)")
    ap.add_argument("--n-new", type=int, default=None,
                    help="decode tokens (default: the model's configured count)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--copy", default="auto", choices=["auto", "on", "off"],
                    help="context-copy proposals (auto: on for the Ouro-2.6B workload)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
