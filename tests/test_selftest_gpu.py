"""Failure detection without a GPU fault: a pipeline wait that nothing
releases gives up after its bound (~1 s), the kernel reports DEV_TIMEOUT
(status 1) and returns, and the context stays usable -- the next kernel
runs and a decode afterwards still matches the full-depth decode."""
import pytest

import synthetic as syn

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_the_context_survives():
    from looped_transformer_self_b200.binding import Decoder, selftest_wait
    r = selftest_wait()
    assert r["status"] == 1 and r["context_alive"]
    assert 200 <= r["wait_ms"] <= 5000, r
    cfg = syn.MODELS["tiny"]
    dec = syn.DECODES["tiny_greedy"]
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny")
    g = Decoder(cfg, dec, w, max_branches=8, max_ctx=128)
    g.prefill(prompt)
    sp, _ = g.generate(16)
    g.prefill(prompt)
    ar, _ = g.generate(16, ar=True)
    g.close()
    assert sp == ar
