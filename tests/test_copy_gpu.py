"""GPU parity of the context-copy proposals (CopyLoop card: copied
continuations screened at depth d1, verified at full depth; readings in
oracle/copy.py) against the oracle, through the C ABI.

Tiny fp32 model (split-tf32 GEMMs, logits within 1e-4 relative of the
oracle): committed tokens, commit sources and steps, per-step branch rows and
the copy statistics are bit-exact.  The screen compares an fp32 softmax
probability with tau on the device and an fp64 one in the oracle, so every
score the oracle evaluated must be more than 1e-3 (relative) away from tau,
else the runs may legitimately differ.  Greedy speculative decoding with
copies equals full-depth greedy decoding on the device, bit for bit.
"""
import numpy as np
import pytest

import synthetic as syn

pytestmark = pytest.mark.gpu

C = 32


def _oracle(cfg, w, prompt, dec, n, tau, reserve):
    from oracle import decode as D
    from oracle.model import LoopedModel
    cp = D.CopyConfig(tau=tau, table=C, reserve=reserve)
    sd = D.SpecDecoder(D.OracleRows(LoopedModel(cfg, w, 512)), prompt, cfg.R, dec.d1, dec.d2, n,
                       dec.temperature, dec.top_p, dec.seed, 512, copy=cp)
    res = sd.run()
    for s in sd.copy_scores:
        assert abs(s - tau) > 1e-3 * max(tau, 1e-12) or tau == 0.0, (s, tau)
    return res


def _gpu(cfg, w, prompt, dec, n, tau, reserve, ar=False):
    from looped_transformer_self_b200.binding import CopyConfig, Decoder
    g = Decoder(cfg, dec, w, max_branches=C, max_ctx=len(prompt) + n + 48, trace_steps=8 * n,
                copy=CopyConfig(tau=tau, reserve=reserve))
    first, _, _ = g.prefill(prompt)
    toks, st = g.generate(n, ar=ar)
    out = ([first] + toks, st)
    if not ar:
        out += (g.read_log(n), g.read_trace(st["steps"]))
    g.close()
    return out


def _repeat_prompt(cfg):
    p = syn.prompt_for("tiny")
    return np.concatenate([p[:20], p[:20], p[:12]]).astype(np.int32)


@pytest.mark.parametrize("tau,reserve,prompt_kind", [(0.0, 7, "plain"), (0.0, 4, "repeat"),
                                                     (0.004, 4, "repeat")])
def test_tiny_greedy_copy_matches_oracle(tau, reserve, prompt_kind):
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny") if prompt_kind == "plain" else _repeat_prompt(cfg)
    dec = syn.DECODES["tiny_greedy"]
    n = 64
    o = _oracle(cfg, w, prompt, dec, n, tau, reserve)
    toks, st, (_, src, step), trace = _gpu(cfg, w, prompt, dec, n, tau, reserve)
    assert toks == o.tokens
    assert src == o.src and step == o.commit_step
    assert trace == o.trace
    for k in ("copy_chains", "copy_rows", "copy_cut", "n_copy", "n_first", "n_second",
              "n_fallback", "gate_checks", "gate_opens"):
        assert st[k] == getattr(o.stats, k), k
    assert o.stats.copy_chains > 0
    ar, _ = _gpu(cfg, w, prompt, dec, n, tau, reserve, ar=True)
    assert toks == ar


def test_tiny_sampled_copy_matches_oracle():
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = _repeat_prompt(cfg)
    dec = syn.DECODES["tiny_sample"]
    n = 48
    o = _oracle(cfg, w, prompt, dec, n, 0.0, 4)
    toks, st, (_, src, step), trace = _gpu(cfg, w, prompt, dec, n, 0.0, 4)
    assert toks == o.tokens
    assert src == o.src and step == o.commit_step
    assert trace == o.trace
    assert st["copy_chains"] == o.stats.copy_chains and st["n_copy"] == o.stats.n_copy
    assert o.stats.copy_chains > 0


def test_bf16_greedy_copy_equals_full_depth_on_device():
    """A bf16 model with head size 128 whose greedy output falls into a loop:
    copied chains are accepted and commit several tokens in one step, and
    the output is the full-depth greedy output bit for bit."""
    from looped_transformer_self_b200.binding import CopyConfig, Decoder
    cfg = syn.ModelConfig("bf16_hd128", "bf16", 256, 2, 128, 512, 1000, 0, 3, 0, 4,
                          resid_scale=0.5, head_gain=4.0, seed=7)
    w = syn.make_weights(cfg)
    base = syn.uniform_prompt(24, cfg.vocab, seed=5)
    prompt = np.concatenate([base, base, base[:8]]).astype(np.int32)
    dec = syn.DecodeConfig(1, 2, 0.0, 1.0, 3, 160)
    n = 160

    def run(ar, copy):
        g = Decoder(cfg, dec, w, max_branches=C, max_ctx=len(prompt) + n + 48,
                    copy=CopyConfig(tau=0.0, reserve=8) if copy else None)
        g.prefill(prompt)
        toks, st = g.generate(n, ar=ar)
        g.close()
        return toks, st

    ar, _ = run(True, False)
    sp, st = run(False, True)
    plain, _ = run(False, False)
    assert sp == ar == plain
    assert st["copy_chains"] > 0
