"""GPU tests of the persistent shared-block pass kernel (opt-in, LT_PASS=1).

The pass kernel runs every layer of a decode pass in one cooperative launch
with the multi-kernel pass's stream-K plans, tile reductions and attention
items, so both paths must produce the same bits: the same tokens, the same
per-step branch rows, and bit-identical readout logits.
"""
import os

import numpy as np
import pytest

import synthetic as syn

pytestmark = pytest.mark.gpu

SMALL_BF16_128 = syn.ModelConfig("bf16_hd128", "bf16", 256, 2, 128, 512, 1000, 0, 3, 0, 4,
                                 resid_scale=0.5, head_gain=4.0, seed=7)
SMALL_BF16_96 = syn.ModelConfig("bf16_hd96", "bf16", 192, 2, 96, 384, 700, 1, 2, 1, 6,
                                resid_scale=0.5, head_gain=4.0, seed=8)


def _run(cfg, dec, w, prompt, use_pass, max_branches, n, max_ctx=None):
    from looped_transformer_self_b200.binding import Decoder
    old = os.environ.get("LT_PASS")
    os.environ["LT_PASS"] = "1" if use_pass else "0"
    try:
        g = Decoder(cfg, dec, w, max_branches=max_branches,
                    max_ctx=max_ctx or len(prompt) + n + 16, trace_steps=8 * n)
    finally:
        if old is None:
            del os.environ["LT_PASS"]
        else:
            os.environ["LT_PASS"] = old
    g.prefill(prompt)
    toks, st = g.generate(n)
    trace = g.read_trace(st["steps"])
    ro = g.read_readouts()
    g.close()
    return toks, st, trace, ro


@pytest.mark.parametrize("cfg,d12,C", [(SMALL_BF16_128, (2, 3), 8), (SMALL_BF16_128, (1, 2), 16),
                                       (SMALL_BF16_96, (2, 3), 16)])
def test_pass_kernel_matches_multi_kernel_bitwise(cfg, d12, C):
    n = 40
    dec = syn.DecodeConfig(d12[0], d12[1], 0.0, 1.0, 3, n)
    w = syn.make_weights(cfg)
    prompt = syn.uniform_prompt(150, cfg.vocab, seed=11)
    a = _run(cfg, dec, w, prompt, True, C, n)
    b = _run(cfg, dec, w, prompt, False, C, n)
    assert a[0] == b[0]
    assert a[1] == b[1]
    assert a[2] == b[2]
    for x, y in zip(a[3], b[3]):
        np.testing.assert_array_equal(np.asarray(x), np.asarray(y))


def test_pass_kernel_sampled_matches_multi_kernel():
    cfg = SMALL_BF16_128
    n = 32
    dec = syn.DecodeConfig(1, 2, 1.0, 0.9, 5, n)
    w = syn.make_weights(cfg)
    prompt = syn.uniform_prompt(100, cfg.vocab, seed=12)
    a = _run(cfg, dec, w, prompt, True, 16, n)
    b = _run(cfg, dec, w, prompt, False, 16, n)
    assert a[0] == b[0] and a[1] == b[1] and a[2] == b[2]


def test_pass_kernel_matches_register_attention_path():
    """Caches sized beyond the ring-buffered attention's limit send the
    multi-kernel pass to the register attention kernel; the pass kernel runs
    the same attention item, so the bits still agree."""
    cfg = SMALL_BF16_128
    n = 24
    dec = syn.DecodeConfig(1, 2, 0.0, 1.0, 3, n)
    w = syn.make_weights(cfg)
    prompt = syn.uniform_prompt(120, cfg.vocab, seed=13)
    a = _run(cfg, dec, w, prompt, True, 16, n, max_ctx=4096)
    b = _run(cfg, dec, w, prompt, False, 16, n, max_ctx=4096)
    assert a[0] == b[0] and a[1] == b[1] and a[2] == b[2]
    for x, y in zip(a[3], b[3]):
        np.testing.assert_array_equal(np.asarray(x), np.asarray(y))
