"""Full-size parity on sampled outputs: the Ouro-1.4B-shaped model of the
benchmark (bf16, 24 shared layers x R = 4, d 2048, 16 x 128 heads, ffn 5632,
vocab 49152), in the benchmark's launch configuration (16-entry branch table,
proposals at depths 1 and 2), on a short prefix the oracle can follow.

* prefill readout logits at depths 1, 2, 4 of the last prompt positions within
  relative L-inf 2e-2 of the oracle (bf16 tolerance);
* greedy pipelined speculative decoding: tokens equal to the oracle's wherever
  the oracle's top-1 / top-2 margin exceeds 0.05, and equal to GPU full-depth
  AR bit for bit.
"""
import numpy as np
import pytest

import synthetic as syn

pytestmark = pytest.mark.gpu


def _margin(z):
    p = np.exp(z - z.max())
    p /= p.sum()
    s = np.sort(p)[::-1]
    return s[0] - s[1]


@pytest.fixture(scope="module")
def ouro():
    cfg = syn.MODELS["ouro14"]
    return cfg, syn.make_weights(cfg)


def test_ouro14_prefill_and_greedy_decode_match_oracle(ouro):
    from looped_transformer_self_b200.binding import Decoder
    from oracle import decode as D
    from oracle.model import LoopedModel
    cfg, w = ouro
    prompt = syn.prompt_for("ouro14")[:8]
    n = 6
    dec = syn.DECODES["ouro14_greedy"].replace(max_new=n)
    g = Decoder(cfg, dec, w, max_branches=16, max_ctx=64)
    first, am, lg = g.prefill(prompt, argmax=True, logits=True)
    lg = lg.cpu().numpy()
    sp = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, 64)), prompt, cfg.R, dec.d1, dec.d2, n,
                       0.0, 1.0, dec.seed, 64, keep_logits=True)
    for pos in (len(prompt) - 2, len(prompt) - 1):
        for t, r in enumerate((1, 2, 4)):
            z = sp.logits[(pos, r)]
            err = np.max(np.abs(lg[pos, t] - z)) / np.max(np.abs(z))
            assert err < 2e-2, (pos, r, err)
    toks, st = g.generate(n)
    g.prefill(prompt)
    ar, _ = g.generate(n, ar=True)
    assert toks == ar  # GPU speculative greedy == GPU full-depth greedy, bit for bit
    gpu = [first] + toks
    for k, (a, b) in enumerate(zip(gpu, sp.tokens)):
        if a != b:
            pos = len(prompt) - 1 + k
            assert _margin(sp.logits[(pos, cfg.R)]) <= 0.05, (k, a, b)
            break


WIDE = syn.ModelConfig("bf16_wide", "bf16", 2048, 16, 128, 5632, 8192, 0, 2, 0, 2,
                       resid_scale=0.0137, head_gain=4.942, seed=11)


def test_full_width_layers_multi_split_context_match_oracle():
    """The Ouro layer shapes (d 2048, 16 x 128 heads, ffn 5632, bf16) with two
    shared layers at R = 2 and a 400-token prompt, so attention runs 4 splits
    per row spread over several blocks at the benchmark's widths: prefill
    readout logits at positions in every split and at both depths within
    relative L-inf 2e-2 of the oracle; greedy speculative decoding equal to GPU
    full-depth AR bit for bit, and to the oracle wherever the oracle's top-1 /
    top-2 margin exceeds 0.05."""
    from looped_transformer_self_b200.binding import Decoder
    from oracle import decode as D
    from oracle.model import LoopedModel
    cfg = WIDE
    w = syn.make_weights(cfg)
    prompt = syn.uniform_prompt(400, cfg.vocab, seed=12)
    n = 4
    dec = syn.DecodeConfig(1, 0, 0.0, 1.0, 5, n)
    g = Decoder(cfg, dec, w, max_branches=16, max_ctx=len(prompt) + 16)
    first, _, lg = g.prefill(prompt, logits=True)
    lg = lg.cpu().numpy()
    sp = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, len(prompt) + 16)), prompt, cfg.R, dec.d1,
                       dec.d2, n, 0.0, 1.0, dec.seed, len(prompt) + 16, keep_logits=True)
    for pos in (5, 130, 257, 399):
        for t, r in enumerate((1, 2)):
            z = sp.logits[(pos, r)]
            err = np.max(np.abs(lg[pos, t] - z)) / np.max(np.abs(z))
            assert err < 2e-2, (pos, r, err)
    toks, _ = g.generate(n)
    g.prefill(prompt)
    ar, _ = g.generate(n, ar=True)
    assert toks == ar
    gpu = [first] + toks
    for k, (a, b) in enumerate(zip(gpu, sp.tokens)):
        if a != b:
            pos = len(prompt) - 1 + k
            assert _margin(sp.logits[(pos, cfg.R)]) <= 0.05, (k, a, b)
            break
    g.close()
