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


# ---------------------------------------------------------------------------
# calibration of the screen (lt_copy_screen_scores) against oracle/copy.py
# ---------------------------------------------------------------------------

def _copy_text(seed, n0=60, vocab=7):
    rng = np.random.default_rng(seed)
    seq = list(rng.integers(0, vocab, size=n0))
    for _ in range(8):  # paste earlier spans: long matches, ties between sources
        a = int(rng.integers(0, len(seq) - 10))
        seq += seq[a:a + int(rng.integers(4, 14))] + [int(rng.integers(0, vocab))]
    return np.asarray(seq, dtype=np.int32)


def _ambiguous(z, T, top_p, eps):
    from oracle import sampling as S
    if top_p >= 1.0 or T == 0.0:
        return False
    p = S.process(z, T, 1.0)
    c = np.cumsum(np.sort(p)[::-1])
    k = int(np.searchsorted(c, top_p, side="left"))
    lo = c[k - 1] if k > 0 else 0.0
    return c[k] - top_p < eps or top_p - lo < eps


@pytest.mark.parametrize("k,cap", [(4, 64), (2, 6)])
@pytest.mark.parametrize("T,top_p", [(0.0, 1.0), (1.0, 1.0), (1.0, 0.9), (0.7, 0.95)])
def test_copy_screen_scores_match_oracle(k, cap, T, top_p):
    """Per position of a copy-rich text: the device's first copied token is
    the oracle lookup's (bit-exact), its depth-d1 screen score is the oracle's
    fp64 softmax within 1e-5 relative, and its full-depth acceptance equals the
    oracle's argmax test (T = 0) or processed p_R (within 2e-6; positions whose
    top-p cut is within 2e-6 of a boundary are skipped, >= 80 % remain)."""
    import torch
    from looped_transformer_self_b200.binding import copy_screen_scores
    from oracle import copy as CP
    from oracle import sampling as S
    seq = _copy_text(k * 10 + cap)
    n, V = len(seq), 1000
    rng = np.random.default_rng(n + V)
    z = (2.5 * rng.standard_normal((n, 2, V))).astype(np.float32)
    for t in range(n - 1):  # full depth sometimes agrees with the next token
        if rng.uniform() < 0.4:
            z[t, 1, seq[t + 1]] += 6.0
    dz = torch.from_numpy(z).cuda()
    tok, score, acc = copy_screen_scores(torch.from_numpy(seq).cuda(), dz[:, 0], dz[:, 1], k, cap,
                                         T, top_p)
    tok, score, acc = tok.cpu().numpy(), score.cpu().numpy(), acc.cpu().numpy()
    found = used = 0
    for t in range(n):
        _, _, prop = CP.lookup(list(seq[:t + 1]), t + 1, k, 16, cap)
        if not prop:
            assert tok[t] == -1 and score[t] == -1.0 and acc[t] == 0.0
            continue
        found += 1
        s = prop[0]
        assert tok[t] == s, t
        z1, zR = z[t, 0].astype(np.float64), z[t, 1].astype(np.float64)
        assert score[t] == pytest.approx(CP.screen_score(z1, s), rel=1e-5)
        if T == 0.0:
            assert acc[t] == (1.0 if int(np.argmax(zR)) == s else 0.0)
            used += 1
        elif not _ambiguous(zR, T, top_p, 2e-6):
            assert abs(acc[t] - S.process(zR, T, top_p)[s]) < 2e-6
            used += 1
    assert found > 20 and used >= 0.8 * found


def test_copy_screen_scores_empty_and_bad_arguments():
    import torch
    from looped_transformer_self_b200 import binding as B
    L = B.lib()
    s = torch.cuda.current_stream().cuda_stream
    t = torch.zeros(4, dtype=torch.int32, device="cuda")
    z = torch.zeros(4, 8, device="cuda")
    o = torch.zeros(4, device="cuda")
    ok = (t.data_ptr(), 4, 2, 8, z.data_ptr(), 8, z.data_ptr(), 8, 8, 1.0, 0.9, t.data_ptr(),
          o.data_ptr(), o.data_ptr(), s)
    assert L.lt_copy_screen_scores(*ok) == 0
    assert L.lt_copy_screen_scores(t.data_ptr(), 0, 2, 8, None, 8, None, 8, 8, 1.0, 0.9, None,
                                   None, None, s) == 0  # empty text
    for i, bad in ((2, 0), (3, 1), (5, 4), (9, -1.0), (10, 0.0), (10, 1.5), (4, None)):
        args = list(ok)
        args[i] = bad
        assert L.lt_copy_screen_scores(*args) == -1, (i, bad)
    torch.cuda.synchronize()


class _FakeDecoder:
    """Stands in for binding.Decoder in calibration: prefill returns fixed
    readout logits [n][n_tags][V] on the device."""

    def __init__(self, cfg, dec, z):
        import torch
        self.cfg, self.dec, self.z = cfg, dec, z
        self.stream = torch.cuda.Stream()

    def prefill(self, tokens, argmax=False, logits=False):
        import torch
        assert logits and len(tokens) == self.z.shape[0]
        return 0, None, torch.from_numpy(self.z.copy()).cuda()


@pytest.mark.parametrize("kind", ["tiny_greedy", "tiny_sample"])
def test_calibration_matches_oracle(kind):
    """copyloop.calibrate on fixed readout logits (device lookup, scores and
    acceptances; host threshold) picks the oracle's tau
    (oracle.copy.prompt_calibration) and admits the same proposals."""
    from looped_transformer_self_b200 import copyloop as CL
    from oracle import copy as CP
    cfg = syn.MODELS["tiny"]
    dec = syn.DECODES[kind]  # readout depths 2, 3, 4
    rng = np.random.default_rng(8)
    base = list(rng.integers(0, 12, size=30))
    prompt = np.array(base + base[:20] + base[5:25], dtype=np.int32)
    P, V = len(prompt), cfg.vocab
    z = rng.normal(size=(P, 3, V)).astype(np.float32)
    for t in range(P - 1):  # full depth agrees with the copied continuation at some positions
        if rng.uniform() < 0.5:
            z[t, 2, prompt[t + 1]] += 8.0
            z[t, 0, prompt[t + 1]] += rng.uniform(0.0, 6.0)
    got = CL.calibrate(_FakeDecoder(cfg, dec, z), prompt)
    tau, scores, acc = CP.prompt_calibration(prompt, z[:, 0].astype(np.float64),
                                             z[:, 2].astype(np.float64), 4, 16, 64,
                                             greedy=dec.temperature == 0.0,
                                             temperature=max(dec.temperature, 1e-9),
                                             top_p=dec.top_p)
    assert got["proposals"] == len(scores) > 10
    assert got["tau"] == pytest.approx(tau, rel=1e-5)
    assert got["admitted"] == int(np.sum(np.asarray(scores) >= tau))
