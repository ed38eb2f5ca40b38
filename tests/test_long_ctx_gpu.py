"""GPU parity of the long-context attention path against the oracle.

Attention streams each block's share of (head, row, 128-position split) units
through a shared-memory ring; long contexts (the Ouro-2.6B prompts, the long
rows of the block-step sweep) spread one row's splits over many blocks.  Each
loop depth attends only to its own cache plane (LoopSpec page, section 2.1
and Fig. 2); attention over a long prefix is split into 128-position pieces
whose partial softmax states are merged.  Checked here through the C ABI:
  * one mixed-depth shared-block pass (lt_block_pass) with attended lengths of
    3100-4200 positions (25-33 splits), permuted slots and mixed depths, head
    sizes 128 and 96, against the oracle's fp64 layer at the bf16 tolerance
    (relative L-inf 2e-2);
  * batch invariance: a row's result does not depend on which other rows share
    the pass (the work assignment of its splits to blocks changes with them;
    the per-split arithmetic and the split-order merge do not), bit for bit;
  * the tiny fp32 model decoding after a 1200-token prompt with max_ctx 4096:
    prefill logits within 1e-4 of the oracle at sampled positions, and the
    greedy decode's integer work (branch rows, slots, sources, steps)
    bit-exact, as for the short-context path.
"""
import numpy as np
import pytest
import torch

import synthetic as syn

pytestmark = pytest.mark.gpu

HD128 = syn.ModelConfig("bf16_hd128", "bf16", 256, 2, 128, 512, 1000, 0, 3, 0, 4,
                        resid_scale=0.5, head_gain=4.0, seed=7)
HD96 = syn.ModelConfig("bf16_hd96", "bf16", 192, 2, 96, 384, 700, 1, 2, 1, 6,
                       resid_scale=0.5, head_gain=4.0, seed=8)


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


def _fill(g, cfg, depth, nslots):
    pool, p0 = g.kv_pool()
    kvs = {}
    for l in range(cfg.n_core):
        for r in sorted(set(depth.tolist())):
            k = syn.random_kv(nslots, cfg.d_model, seed=1000 + 10 * l + r)
            v = syn.random_kv(nslots, cfg.d_model, seed=2000 + 10 * l + r)
            kvs[(l, r)] = (k, v)
            plane = p0 + l * cfg.R + (r - 1)
            pool[plane, :nslots, 0] = torch.from_numpy(k).to(pool.dtype).to(pool.device)
            pool[plane, :nslots, 1] = torch.from_numpy(v).to(pool.dtype).to(pool.device)
    return kvs


def _pass(cfg, w, depth, lens, lists, offs, nslots, max_ctx, hid0):
    from looped_transformer_self_b200.binding import Decoder
    # workspace of NaN / -1 bytes: nothing may be read before it is written
    g = Decoder(cfg, syn.DecodeConfig(1, 2, 0.0, 1.0, 2, 4), w, max_branches=8, max_ctx=max_ctx,
                workspace_fill=0xFF)
    kvs = _fill(g, cfg, depth, nslots)
    hid = torch.from_numpy(hid0).cuda()
    g.block_pass(depth, lens, torch.from_numpy(lists).cuda(), offs, hid)
    g.close()
    return hid.cpu().numpy(), kvs


@pytest.mark.parametrize("cfg", [HD128, HD96], ids=["hd128", "hd96"])
def test_long_context_block_pass_matches_oracle(cfg):
    from oracle.model import LoopedModel
    depth = np.array([1, 2, 3, 4, 2, 1], np.int32)
    lens = np.array([3100, 3650, 4200, 3333, 3901, 4097], np.int32)[: len(depth)]
    lists, offs, nslots = _layout(depth, lens, seed=21)
    w = syn.make_weights(cfg)
    hid0 = syn.random_hidden(len(depth), cfg.d_model, seed=6)
    got, kvs = _pass(cfg, w, depth, lens, lists, offs, nslots, nslots + 64, hid0)
    assert lens.min() > 24 * 128  # 25-33 splits per row, spread over many blocks
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


@pytest.mark.parametrize("cfg", [HD128, HD96], ids=["hd128", "hd96"])
def test_rows_are_batch_invariant_bitwise(cfg):
    """The same rows alone and among others (different split-to-block
    assignments, the same cache contents): identical bits per row."""
    depth = np.array([1, 3, 2, 2, 1][: 5 if cfg.R >= 3 else 4], np.int32)
    lens = np.array([4100, 1500, 2047, 130, 3333][: len(depth)], np.int32)
    lists, offs, nslots = _layout(depth, lens, seed=5)
    w = syn.make_weights(cfg)
    hid0 = syn.random_hidden(len(depth), cfg.d_model, seed=9)
    full, _ = _pass(cfg, w, depth, lens, lists, offs, nslots, nslots + 64, hid0)
    for sub in ([1], [0, 4], [3, 2]):
        sl = [lists[offs[r]:offs[r] + lens[r] + 1] for r in sub]
        so = np.cumsum([0] + [len(x) for x in sl[:-1]]).astype(np.int32)
        got, _ = _pass(cfg, w, depth[sub], lens[sub], np.concatenate(sl), so, nslots, nslots + 64,
                       np.ascontiguousarray(hid0[sub]))
        np.testing.assert_array_equal(got, full[sub])


def test_tiny_long_prompt_decode_matches_oracle():
    """Tiny fp32 model, 1200-token prompt, max_ctx 4096 (10-11 attention
    splits per row, fp32 cache path): prefill logits at sampled positions and
    every readout depth within 1e-4 of the oracle; greedy speculative decoding
    equals GPU AR and its integer work is bit-exact against the oracle."""
    from oracle import decode as D
    from oracle.model import LoopedModel
    from test_decode_gpu import TOL_F32, _rel_linf, check_integer_work
    from looped_transformer_self_b200.binding import Decoder
    cfg = syn.MODELS["tiny"]
    w = syn.make_weights(cfg)
    prompt = syn.uniform_prompt(1200, cfg.vocab, seed=13)
    dec = syn.DECODES["tiny_greedy"].replace(max_new=24)
    g = Decoder(cfg, dec, w, max_branches=8, max_ctx=4096, trace_steps=256)
    first, _, lg = g.prefill(prompt, logits=True)
    lg = lg.cpu().numpy()
    sp_o = D.decode_spec(D.OracleRows(LoopedModel(cfg, w, 1300)), prompt, cfg.R, dec.d1, dec.d2,
                         dec.max_new, 0.0, 1.0, dec.seed, 1300, keep_logits=True)
    tags = [2, 3, 4]
    for pos in list(range(0, 1200, 97)) + [1199]:
        for t, r in enumerate(tags):
            assert _rel_linf(lg[pos, t], sp_o.logits[(pos, r)]) < TOL_F32, (pos, r)
    assert first == sp_o.tokens[0]
    g.prefill(prompt)
    sp_toks, st = g.generate(dec.max_new)
    g.prefill(prompt)
    ar_toks, _ = g.generate(dec.max_new, ar=True)
    assert sp_toks == ar_toks
    g.prefill(prompt)
    sp_toks, st = g.generate(dec.max_new)
    _, src, step = g.read_log(dec.max_new)
    low = check_integer_work(g, sp_o, st, src, step)
    if low is None:
        assert [first] + sp_toks == sp_o.tokens
    g.close()
