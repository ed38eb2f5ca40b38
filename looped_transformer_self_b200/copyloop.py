"""Calibration of the copy screen threshold on the prompt.

CopyLoop card (kongchang.com): copied continuations are scored at a shallow
loop depth, and the threshold that admits them to full-depth verification
comes from a light calibration.  The decoder's copy proposals (lt_decode_config
copy_* fields) use, for the prefix ending at position t, the longest earlier
backward match (>= k tokens, capped at match_cap; the most recent on ties) in
the committed context and the committed tokens after it.  On the prompt every
position is committed, so for each prompt position t with a proposal the
library (lt_copy_screen_scores) gives its first copied token s, its screen
score (softmax at T = 1 of the depth-d1 readout of t, at s) and whether full
depth accepts it (greedy: the depth-R argmax is s; sampling: with probability
p_R(s) under the decode's temperature and top-p); this module picks the
threshold tau that maximises the sum over admitted proposals of
(2 accept - 1): a proposal is admitted when it is more likely accepted than
rejected.  With no proposal, tau = 1.

The card does not say what text the calibration reads.  The prompt alone can
hold no copy the model would accept (a model that does not continue copied
spans, such as a random-init one, still repeats its own output), so
`calibrate(..., warm=N)` appends N tokens the decoder generates from it; the
benchmark calibrates on a separate prompt of the same workload, never on the
text it times.
"""
from __future__ import annotations

from typing import Dict, Sequence

import numpy as np


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
    prefill with readout logits (resets the decoder's state), then
    lt_copy_screen_scores on the device gives every position's first copied
    token, its screen score and its full-depth acceptance; only the choice of
    tau from those host arrays happens here.  warm > 0: the calibration text
    is the prompt followed by `warm` tokens that the decoder generates from it
    first (its own continuation -- copies recur in generated text as much as
    in prompts)."""
    import torch

    from .binding import copy_screen_scores
    cfg, dec = decoder.cfg, decoder.dec
    prompt = np.asarray(prompt, dtype=np.int32)
    if warm > 0:
        first, _, _ = decoder.prefill(prompt)
        toks, _ = decoder.generate(warm)
        prompt = np.concatenate([prompt, np.asarray([first] + toks, dtype=np.int32)])
    _, _, lg = decoder.prefill(prompt, logits=True)  # [P][n_tags][V]
    tags = sorted({r for r in (dec.d1, dec.d2, cfg.R) if r > 0})
    d_tok = torch.from_numpy(prompt).to(lg.device)
    with torch.cuda.stream(decoder.stream):
        tok, score, acc = copy_screen_scores(d_tok, lg[:, tags.index(dec.d1)],
                                             lg[:, tags.index(cfg.R)], k, match_cap,
                                             dec.temperature, dec.top_p, stream=decoder.stream)
    decoder.stream.synchronize()
    tok, score, acc = tok.cpu().numpy(), score.cpu().numpy(), acc.cpu().numpy()
    del lg
    has = tok >= 0
    if not has.any():
        return {"tau": 1.0, "text_len": int(len(prompt)), "proposals": 0, "admitted": 0,
                "accept_rate": 0.0}
    scores, accs = score[has].astype(np.float64), acc[has].astype(np.float64)
    tau = threshold(scores, accs)
    keep = scores >= tau
    return {"tau": tau, "text_len": int(len(prompt)), "proposals": int(has.sum()),
            "admitted": int(keep.sum()),
            "accept_rate": float(accs.mean()),
            "accept_rate_admitted": float(accs[keep].mean()) if keep.any() else 0.0}
