"""GPU parity of one mixed-depth shared-block pass (lt_block_pass) against the
oracle: rows at different loop depths, each with its own randomly permuted
cache slots and a context spanning several attention splits, caches filled
from seeded host data (synthetic.random_kv) on both sides."""
import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu

CFG = syn.ModelConfig("bf16_hd128", "bf16", 256, 2, 128, 512, 1000, 0, 3, 0, 4,
                      resid_scale=0.5, head_gain=4.0, seed=7)


def _layout(depth, lens, seed):
    """Disjoint slot ranges per depth; each row's list is a permutation of its range."""
    rng = np.random.default_rng(seed)
    nxt, lists, offs = {}, [], []
    for r, l in zip(depth, lens):
        start = nxt.get(r, 0)
        nxt[r] = start + l + 1
        offs.append(sum(len(x) for x in lists))
        lists.append(rng.permutation(np.arange(start, start + l + 1)).astype(np.int32))
    return np.concatenate(lists), np.array(offs, np.int32), max(nxt.values())


@pytest.mark.parametrize("cfg", [CFG])
def test_block_pass_matches_oracle(cfg):
    from looped_transformer_self_b200.binding import Decoder
    from oracle.model import LoopedModel
    depth = np.array([1, 2, 3, 4, 2], np.int32)
    lens = np.array([40, 130, 300, 7, 260], np.int32)  # attended positions 0..len
    lists, offs, nslots = _layout(depth, lens, seed=11)
    w = syn.make_weights(cfg)
    C = 8
    dec = syn.DecodeConfig(1, 2, 0.0, 1.0, 2, 4)
    g = Decoder(cfg, dec, w, max_branches=C, max_ctx=max(nslots, 400))
    pool, p0 = g.kv_pool()
    d = cfg.d_model
    # cache contents for every (core layer, depth) plane that a row reads
    kvs = {}
    for l in range(cfg.n_core):
        for r in sorted(set(depth.tolist())):
            k = syn.random_kv(nslots, d, seed=1000 + 10 * l + r)
            v = syn.random_kv(nslots, d, seed=2000 + 10 * l + r)
            kvs[(l, r)] = (k, v)
            plane = p0 + l * cfg.R + (r - 1)
            pool[plane, :nslots, 0] = torch.from_numpy(k).to(pool.dtype).to(pool.device)
            pool[plane, :nslots, 1] = torch.from_numpy(v).to(pool.dtype).to(pool.device)
    hid0 = syn.random_hidden(len(depth), d, seed=5)
    hid = torch.from_numpy(hid0).cuda()
    g.block_pass(depth, lens, torch.from_numpy(lists).cuda(), offs, hid)
    got = hid.cpu().numpy()
    for i in range(len(depth)):
        m = LoopedModel(cfg, w, nslots)
        for l in range(cfg.n_core):
            K, V = m.cache(f"core{l}", int(depth[i]))
            K[:] = kvs[(l, int(depth[i]))][0]
            V[:] = kvs[(l, int(depth[i]))][1]
        sl = lists[offs[i]:offs[i] + lens[i] + 1].tolist()
        ref = m.iterate(hid0[i].astype(np.float64), int(depth[i]), int(lens[i]), sl)
        err = np.max(np.abs(got[i] - ref)) / np.max(np.abs(ref))
        assert err < 2e-2, (i, err)


def test_block_pass_timed_replays_are_stable():
    """The captured-graph replay path runs and times every replay."""
    from looped_transformer_self_b200.binding import Decoder
    cfg = CFG
    depth = np.array([1, 3], np.int32)
    lens = np.array([20, 50], np.int32)
    lists, offs, nslots = _layout(depth, lens, seed=3)
    g = Decoder(cfg, syn.DecodeConfig(1, 2, 0.0, 1.0, 2, 4), syn.make_weights(cfg), max_branches=8,
                max_ctx=200)
    pool, _ = g.kv_pool()
    pool.copy_(torch.from_numpy(syn.random_kv(pool.numel() // cfg.d_model, cfg.d_model, seed=9))
               .view(pool.shape).to(pool.dtype))
    hid = torch.from_numpy(syn.random_hidden(2, cfg.d_model, seed=1)).cuda()
    ms = g.block_pass(depth, lens, torch.from_numpy(lists).cuda(), offs, hid, iters=5, timed=True)
    assert len(ms) == 5 and all(0 < t < 1000 for t in ms)
    assert torch.isfinite(hid).all()


def test_profile_gemms_times_the_pass_gemms_and_resets_state():
    """lt_profile_gemms replays one pass's shared-block GEMMs as a graph: a
    positive time, the algorithmic bytes of 4 GEMMs per layer, and a decode
    state that must be prefilled again."""
    from looped_transformer_self_b200.binding import Decoder, LoopedSpecError
    cfg = CFG
    C = 8
    g = Decoder(cfg, syn.DecodeConfig(1, 2, 0.0, 1.0, 2, 4), syn.make_weights(cfg), max_branches=C,
                max_ctx=200)
    g.prefill(syn.uniform_prompt(20, cfg.vocab, seed=2))
    r = g.profile_gemms(3)
    d, f = cfg.d_model, cfg.ffn
    want = 0.0
    for n_out, k in ((3 * d, d), (d, d), (2 * f, d), (d, f)):
        want += 2.0 * (n_out * k + C * k) + 4.0 * C * n_out
    assert r["launches"] == 4 * cfg.n_core
    assert abs(r["bytes"] - want * cfg.n_core) < 1.0
    assert 0.0 < r["ms"] < 100.0
    with pytest.raises(LoopedSpecError):
        g.generate(2)
    g.prefill(syn.uniform_prompt(20, cfg.vocab, seed=2))
    toks, _ = g.generate(4)
    assert len(toks) == 4
    g.close()
