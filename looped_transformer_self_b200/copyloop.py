"""Calibration of the copy screen threshold on the prompt.

CopyLoop card (kongchang.com): copied continuations are scored at a shallow
loop depth, and the threshold that admits them to full-depth verification
comes from a light calibration.  The decoder's copy proposals (lt_decode_config
copy_* fields) use, for the prefix ending at position t, the longest earlier
backward match (>= k tokens, capped at match_cap; the most recent on ties) in
the committed context and the committed tokens after it.  On the prompt every
position is committed, so for each prompt position t with a proposal this
module takes its first copied token s, its screen score (softmax at T = 1 of
the depth-d1 readout of t, at s) and whether full depth accepts it (greedy:
the depth-R argmax is s; sampling: with probability p_R(s) under the decode's
temperature and top-p), and picks the threshold tau that maximises the sum
over admitted proposals of (2 accept - 1): a proposal is admitted when it is
more likely accepted than rejected.  With no proposal, tau = 1.

The card does not say what text the calibration reads.  The prompt alone can
hold no copy the model would accept (a model that does not continue copied
spans, such as a random-init one, still repeats its own output), so
`calibrate(..., warm=N)` appends N tokens the decoder generates from it; the
benchmark calibrates on a separate prompt of the same workload, never on the
text it times.
"""
from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

import numpy as np


def first_copies(prompt: Sequence[int], k: int, match_cap: int) -> Dict[int, int]:
    """{t: first copied token} for every prompt position t whose prefix
    prompt[0..t] (all committed) has a copy proposal."""
    seq = np.asarray(prompt, dtype=np.int64)
    n = len(seq)
    ends: Dict[Tuple[int, ...], List[int]] = {}  # k-gram -> end positions so far
    out = {}
    for t in range(k - 1, n):
        key = tuple(seq[t - k + 1:t + 1].tolist())
        best_e, best_m = -1, 0
        # sources: e <= t - 1 (followed by a committed token inside prompt[0..t])
        for e in ends.get(key, ()):
            m = k
            while m < match_cap and m <= e and seq[e - m] == seq[t - m]:
                m += 1
            if m >= best_m:
                best_e, best_m = e, m
        if best_e >= 0:
            out[t] = int(seq[best_e + 1])
        ends.setdefault(key, []).append(t)
    return out


def threshold(scores: Sequence[float], accept: Sequence[float]) -> float:
    """tau maximising sum over score >= tau of (2 accept - 1); the larger tau
    on ties; 1 when no threshold gains."""
    s = np.asarray(scores, np.float64)
    a = np.asarray(accept, np.float64)
    if s.size == 0:
        return 1.0
    order = np.argsort(-s, kind="stable")
    gain = np.cumsum(2.0 * a[order] - 1.0)  # admitting the top j+1 scores
    ss = s[order]
    best_tau, best_gain = 1.0, 0.0
    j = 0
    while j < len(ss):  # group equal scores: a threshold admits all of them
        j2 = j
        while j2 + 1 < len(ss) and ss[j2 + 1] == ss[j]:
            j2 += 1
        if gain[j2] > best_gain:
            best_tau, best_gain = float(ss[j]), float(gain[j2])
        j = j2 + 1
    return best_tau


def calibrate(decoder, prompt, k=4, match_cap=64, warm=0) -> Dict[str, float]:
    """tau for `decoder` (a binding.Decoder whose d1 >= 1) on `prompt`: one
    prefill with readout logits (resets the decoder's state), screen scores
    and full-depth acceptance of every position's first copied token.  warm >
    0: the calibration text is the prompt followed by `warm` tokens that the
    decoder generates from it first (its own continuation -- copies recur in
    generated text as much as in prompts)."""
    import torch

    from .binding import readout_tv
    cfg, dec = decoder.cfg, decoder.dec
    prompt = np.asarray(prompt, dtype=np.int32)
    if warm > 0:
        first, _, _ = decoder.prefill(prompt)
        toks, _ = decoder.generate(warm)
        prompt = np.concatenate([prompt, np.asarray([first] + toks, dtype=np.int32)])
    props = first_copies(prompt, k, match_cap)
    if not props:
        return {"tau": 1.0, "text_len": int(len(prompt)), "proposals": 0, "admitted": 0,
                "accept_rate": 0.0}
    _, _, lg = decoder.prefill(prompt, logits=True)  # [P][n_tags][V]
    tags = sorted({r for r in (dec.d1, dec.d2, cfg.R) if r > 0})
    t_idx = torch.tensor(sorted(props), device=lg.device)
    s_idx = torch.tensor([props[t] for t in sorted(props)], device=lg.device)
    z1 = lg[t_idx, tags.index(dec.d1)]
    zR = lg[t_idx, tags.index(cfg.R)].contiguous()
    rows = torch.arange(len(t_idx), device=lg.device)
    scores = torch.softmax(z1.double(), dim=-1)[rows, s_idx]
    if dec.temperature == 0.0:
        acc = (zR.argmax(dim=-1) == s_idx).double()
    else:
        zb = zR.clone()
        readout_tv(zR, zb, dec.temperature, dec.top_p, stream=decoder.stream)  # zR -> p_R
        decoder.stream.synchronize()
        acc = zR[rows, s_idx].double()
    scores, acc = scores.cpu().numpy(), acc.cpu().numpy()
    del lg
    tau = threshold(scores, acc)
    keep = scores >= tau
    return {"tau": tau, "text_len": int(len(prompt)), "proposals": int(len(scores)),
            "admitted": int(keep.sum()),
            "accept_rate": float(acc.mean()),
            "accept_rate_admitted": float(acc[keep].mean()) if keep.any() else 0.0}
