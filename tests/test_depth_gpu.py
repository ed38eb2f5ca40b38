"""GPU parity of depth selection's measurement (LoopSpec page, section 2.4,
Eq. 7; section 3.1, Fig. 3 right) against the oracle.

lt_readout_tv turns two logit rows into readout distributions with the decode
step's own processing (temperature, top-p, normalisation) and returns their
total variation.  The device works in fp32 and the oracle in fp64, so values
agree to ~1e-5; the top-p cut is an integer decision taken from those floats
(fp32 probabilities carry ~1e-6 absolute error in their cumulative mass), so
rows whose cumulative mass crosses top-p within 2e-6 of a boundary token
(either side) are excluded, and at least 80 % of the rows must remain.
"""
import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu


def _ambiguous(z, T, top_p, eps):
    from oracle import sampling as S
    if top_p >= 1.0 or T == 0.0:
        return False
    p = S.process(z, T, 1.0)
    c = np.cumsum(np.sort(p)[::-1])
    k = int(np.searchsorted(c, top_p, side="left"))
    lo = c[k - 1] if k > 0 else 0.0
    return c[k] - top_p < eps or top_p - lo < eps


@pytest.mark.parametrize("V", [5, 1000, 49152, 65536 + 3])
@pytest.mark.parametrize("T,top_p", [(1.0, 0.7), (0.7, 0.95), (1.0, 1.0), (0.0, 0.7)])
def test_readout_tv_matches_oracle(V, T, top_p):
    from looped_transformer_self_b200.binding import readout_tv
    from oracle import depth as Dp
    from oracle import sampling as S
    rng = np.random.default_rng(V * 7 + int(T * 10) + int(top_p * 100))
    n = 37
    z = (3.0 * rng.standard_normal((n, 2, V))).astype(np.float32)
    # every fifth row pair shares most of its logits (small TV)
    z[::5, 1] = z[::5, 0] + (0.1 * rng.standard_normal((len(z[::5]), V))).astype(np.float32)
    d = torch.from_numpy(z).cuda()
    tv = readout_tv(d[:, 0, :], d[:, 1, :], T, top_p).cpu().numpy()
    proc = d.cpu().numpy()
    used = 0
    for i in range(n):
        za, zb = z[i, 0].astype(np.float64), z[i, 1].astype(np.float64)
        if _ambiguous(za, T, top_p, 2e-6) or _ambiguous(zb, T, top_p, 2e-6):
            continue
        used += 1
        want = Dp.readout_tv(za, zb, T, top_p)
        if T == 0.0:
            assert tv[i] == want
            continue
        assert abs(tv[i] - want) < 1e-5, (i, tv[i], want)
        for k, zk in ((0, za), (1, zb)):
            np.testing.assert_allclose(proc[i, k], S.process(zk, T, top_p), atol=2e-6, rtol=0)
    assert used >= 0.8 * n


def test_readout_tv_empty_and_bad_arguments():
    from looped_transformer_self_b200 import binding as B
    z = torch.zeros(0, 8, device="cuda")
    assert B.readout_tv(z, z, 1.0, 0.7).numel() == 0
    L = B.lib()
    zz = torch.zeros(2, 8, device="cuda")
    out = torch.zeros(2, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert L.lt_readout_tv(zz.data_ptr(), 4, zz.data_ptr(), 8, 2, 8, 1.0, 0.7, out.data_ptr(), s) == -1
    assert L.lt_readout_tv(zz.data_ptr(), 8, zz.data_ptr(), 8, 2, 8, -1.0, 0.7, out.data_ptr(), s) == -1
    assert L.lt_readout_tv(zz.data_ptr(), 8, zz.data_ptr(), 8, 2, 8, 1.0, 0.0, out.data_ptr(), s) == -1
    assert L.lt_readout_tv(None, 8, zz.data_ptr(), 8, 2, 8, 1.0, 0.7, out.data_ptr(), s) == -1


def test_tiny_tv_by_depth_matches_oracle():
    """Per-position TV(p_r, p_R) of the tiny model's prompt, every depth r < R:
    device prefill readouts + lt_readout_tv against the oracle's prefill with
    every depth as a readout depth."""
    from looped_transformer_self_b200 import depth_select as DS
    from oracle import decode as D
    from oracle import depth as Dp
    from oracle.model import LoopedModel
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny")
    dec = syn.DECODES["tiny_sample"]
    depths = DS.default_depths(cfg.R)
    got = DS.measure_tv(cfg, dec, w, prompt, depths, 1.0, 0.7, max_branches=8)
    zs = D.prefill(D.OracleRows(LoopedModel(cfg, w, len(prompt) + 8)), prompt, cfg.R,
                   list(range(1, cfg.R + 1)), keep_logits=True)
    want = Dp.tv_by_depth(zs, range(len(prompt)), depths, cfg.R, 1.0, 0.7)
    for r in depths:
        ok = [t for t in range(len(prompt))
              if not (_ambiguous(zs[(t, r)], 1.0, 0.7, 1e-3) or _ambiguous(zs[(t, cfg.R)], 1.0, 0.7, 1e-3))]
        assert len(ok) >= 0.8 * len(prompt)
        np.testing.assert_allclose(got[r][ok], want[r][ok], atol=2e-3, rtol=0)
    # the envelope of the device means is the oracle's envelope of its own means
    # up to the measurement tolerance
    a, b = DS.envelope(depths, [float(got[r].mean()) for r in depths])
    oa, ob = Dp.fit_envelope(depths, [float(want[r].mean()) for r in depths])
    assert a == pytest.approx(oa, abs=0.05) and b == pytest.approx(ob, rel=0.02)


def test_tiny_depth_selection_runs_end_to_end():
    from looped_transformer_self_b200 import depth_select as DS
    res = DS.run("tiny", n=24, candidates=2, tv_positions=48)
    assert res["depths"] == [1, 2, 3]
    assert all(0.0 <= m <= 1.0 for m in res["mean_tv"])
    pairs = [(p["d1"], p["d2"]) for p in res["sweep"]]
    assert set(pairs) <= set(DS.candidate_pairs(4)) and len(pairs) >= 2
    assert all(p["tok_s"] > 0 for p in res["sweep"]) and res["ar_tok_s"] > 0
    assert tuple(res["measured_best"]) in pairs
