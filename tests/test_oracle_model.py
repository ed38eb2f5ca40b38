"""Pins of the oracle's fp64 model arithmetic.

* closed forms and invariants of RMSNorm, RoPE and softmax attention;
* the looped model equals an unrolled Transformer with tied weights, written
  here as a full-sequence batch computation on PyTorch library primitives
  (F.linear, F.rms_norm, F.scaled_dot_product_attention with a causal mask,
  F.silu) -- which also checks the oracle's incremental, slot-addressed caches
  against a full causal recompute of every prefix;
* s = 0 makes every shared-block iteration the identity (all depths agree);
* cache slots are only addresses: a permutation of them changes nothing.
"""
import ctypes

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import synthetic as syn
from oracle import decode as D
from oracle.model import LoopedModel, lib

dp = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
fp = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
ip = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def test_rmsnorm_closed_form():
    rng = np.random.default_rng(0)
    h = rng.normal(size=64) * 3
    g = np.ones(64, np.float32)
    out = np.empty(64)
    lib().orc_rmsnorm(64, dp(h), fp(g), 0.0, dp(out))
    assert abs(np.sqrt(np.mean(out ** 2)) - 1.0) < 1e-14
    out2 = np.empty(64)
    h2 = h * 17.0
    lib().orc_rmsnorm(64, dp(h2), fp(g), 0.0, dp(out2))
    np.testing.assert_allclose(out, out2, rtol=1e-14)
    g2 = rng.normal(size=64).astype(np.float32)
    out3 = np.empty(64)
    lib().orc_rmsnorm(64, dp(h), fp(g2), 0.0, dp(out3))
    np.testing.assert_allclose(out3, out * g2, rtol=1e-14)


def _rope(v, H, hd, pos, theta=1e4):
    v = v.copy()
    lib().orc_rope(H, hd, pos, theta, dp(v))
    return v


def test_rope_is_a_relative_rotation():
    rng = np.random.default_rng(1)
    H, hd = 2, 16
    q, k = rng.normal(size=H * hd), rng.normal(size=H * hd)
    np.testing.assert_allclose(_rope(q, H, hd, 0), q, rtol=0, atol=0)
    for m in (1, 5, 40):
        np.testing.assert_allclose(np.linalg.norm(_rope(q, H, hd, m)), np.linalg.norm(q), rtol=1e-13)
    # <rope(q, m), rope(k, n)> depends only on m - n, per head
    for m, n in ((7, 3), (30, 26), (4, 0)):
        a = (_rope(q, H, hd, m) * _rope(k, H, hd, n)).reshape(H, hd).sum(1)
        b = (_rope(q, H, hd, m + 11) * _rope(k, H, hd, n + 11)).reshape(H, hd).sum(1)
        np.testing.assert_allclose(a, b, rtol=1e-11)
    # lowest frequency pair (i = 0) rotates by exactly pos radians
    e = np.zeros(hd)
    e[0] = 1.0
    r = _rope(e, 1, hd, 2)
    np.testing.assert_allclose([r[0], r[hd // 2]], [np.cos(2.0), np.sin(2.0)], atol=1e-15)


def test_attention_special_cases():
    rng = np.random.default_rng(2)
    H, hd, d = 2, 8, 16
    K = rng.normal(size=(5, d))
    V = rng.normal(size=(5, d))
    q = rng.normal(size=d)
    out = np.empty(d)
    slots = np.array([3], np.int32)
    lib().orc_attend(H, hd, d, 1, dp(q), dp(K), dp(V), ip(slots), dp(out))
    np.testing.assert_allclose(out, V[3], rtol=1e-15)
    K2 = np.tile(K[0], (5, 1))
    slots = np.array([4, 1, 2], np.int32)
    lib().orc_attend(H, hd, d, 3, dp(q), dp(K2), dp(V), ip(slots), dp(out))
    np.testing.assert_allclose(out, V[[4, 1, 2]].mean(0), rtol=1e-14)


# -- full recompute with library primitives ----------------------------------


def _torch_layer(w, name, x, s, cfg):
    """One layer over a whole sequence x [T, d] (fp64), causal."""
    T, d = x.shape
    H, hd, f = cfg.n_heads, cfg.head_dim, cfg.ffn
    t = lambda k: torch.from_numpy(w[f"{name}.{k}"].astype(np.float64))
    a = F.rms_norm(x, (d,), t("g1"), eps=cfg.rms_eps)
    qkv = F.linear(a, t("wqkv"))
    q, k, v = qkv[:, :d], qkv[:, d:2 * d], qkv[:, 2 * d:]
    pos = torch.arange(T, dtype=torch.float64)[:, None]
    inv = cfg.rope_theta ** (-2.0 * torch.arange(hd // 2, dtype=torch.float64) / hd)
    ang = pos * inv[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rope(u):
        u = u.view(T, H, hd)
        u1, u2 = u[..., :hd // 2], u[..., hd // 2:]
        c, s_ = cos[:, None, :], sin[:, None, :]
        return torch.cat([u1 * c - u2 * s_, u2 * c + u1 * s_], -1)

    qh = rope(q).transpose(0, 1)
    kh = rope(k).transpose(0, 1)
    vh = v.view(T, H, hd).transpose(0, 1)
    o = F.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
    o = o.transpose(0, 1).reshape(T, d)
    x = x + s * F.linear(o, t("wo"))
    a2 = F.rms_norm(x, (d,), t("g2"), eps=cfg.rms_eps)
    gu = F.linear(a2, t("wgu"))
    act = F.silu(gu[:, :f]) * gu[:, f:]
    return x + s * F.linear(act, t("wd"))


def _torch_logits_all_depths(cfg, w, prompt):
    """Unrolled: prelude, then R copies of the shared block (tied weights), and
    at every depth r: coda layers over the depth-r states, norm, head."""
    x = torch.from_numpy(w["embed"][prompt].astype(np.float64))
    for i in range(cfg.n_prelude):
        x = _torch_layer(w, f"pre{i}", x, 1.0, cfg)
    out = {}
    for r in range(1, cfg.R + 1):
        for i in range(cfg.n_core):
            x = _torch_layer(w, f"core{i}", x, cfg.resid_scale, cfg)
        y = x
        for i in range(cfg.n_coda):
            y = _torch_layer(w, f"coda{i}", y, 1.0, cfg)
        y = F.rms_norm(y, (cfg.d_model,), torch.from_numpy(w["final_norm"].astype(np.float64)),
                       eps=cfg.rms_eps)
        out[r] = F.linear(y, torch.from_numpy(w["head"].astype(np.float64))).numpy()
    return out


@pytest.mark.parametrize("model,s", [("tiny", 1.0), ("tiny", 0.5)])
def test_looped_model_equals_unrolled_full_recompute(model, s):
    cfg = syn.MODELS[model].replace(resid_scale=s)
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for(model, 12)
    ref = _torch_logits_all_depths(cfg, w, prompt)
    m = LoopedModel(cfg, w, 16)
    zs = D.prefill(D.OracleRows(m), prompt, cfg.R, list(range(1, cfg.R + 1)), keep_logits=True)
    for (pos, r), z in zs.items():
        np.testing.assert_allclose(z, ref[r][pos], rtol=1e-10, atol=1e-10)


def test_bf16_shapes_against_full_recompute():
    """A small bf16-valued model (no prelude/coda layers, Ouro layout)."""
    cfg = syn.ModelConfig("t", "bf16", 64, 2, 32, 96, 40, 0, 3, 0, 3, resid_scale=0.7)
    w = syn.make_weights(cfg)
    prompt = syn.zipf_prompt(9, cfg.vocab)
    ref = _torch_logits_all_depths(cfg, w, prompt)
    m = LoopedModel(cfg, w, 16)
    zs = D.prefill(D.OracleRows(m), prompt, cfg.R, [1, 2, 3], keep_logits=True)
    for (pos, r), z in zs.items():
        np.testing.assert_allclose(z, ref[r][pos], rtol=1e-10, atol=1e-10)


def test_zero_residual_scale_makes_all_depths_agree():
    cfg = syn.MODELS["tiny"].replace(resid_scale=0.0)
    m = LoopedModel(cfg, syn.make_weights(cfg), 16)
    prompt = syn.prompt_for("tiny", 6)
    zs = D.prefill(D.OracleRows(m), prompt, cfg.R, [1, 2, 3, 4], keep_logits=True)
    for pos in range(6):
        for r in (2, 3, 4):
            np.testing.assert_array_equal(zs[(pos, r)], zs[(pos, 1)])


def test_slot_permutation_changes_nothing():
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = syn.prompt_for("tiny", 7)
    rows1 = D.OracleRows(LoopedModel(cfg, w, 32))
    rows2 = D.OracleRows(LoopedModel(cfg, w, 32))
    perm = np.random.default_rng(0).permutation(32)[:7]
    for pos in range(7):
        prefix = list(prompt[:pos + 1])
        h1 = rows1.prelude(prefix, pos, list(range(pos + 1)))
        h2 = rows2.prelude(prefix, pos, [int(x) for x in perm[:pos + 1]])
        for r in range(1, 5):
            h1 = rows1.iterate(h1, r, prefix, pos, list(range(pos + 1)))
            h2 = rows2.iterate(h2, r, prefix, pos, [int(x) for x in perm[:pos + 1]])
        np.testing.assert_array_equal(h1, h2)
        np.testing.assert_array_equal(rows1.readout(h1, 4, prefix, pos, list(range(pos + 1))),
                                      rows2.readout(h2, 4, prefix, pos, [int(x) for x in perm[:pos + 1]]))
