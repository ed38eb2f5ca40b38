"""fp64 looped-Transformer model for the oracle (test infrastructure only).

Eq. 1 of the LoopSpec page (section 2.1): H^(0) = P(X), H^(r) = B(H^(r-1)),
p_r = C(H^(r)), 1 <= r <= R.  Caches (section 2.1 / Fig. 2, section 2.4):
  * the prelude layers keep one cache (the prelude does not depend on depth);
  * shared-block layer l at loop iteration r reads and writes only the cache of
    (l, r): states of different depths are never mixed;
  * coda layers keep one cache per readout depth r (a readout at depth r runs
    the coda over the depth-r state; reading: the coda cache is tagged by the
    readout depth, the only reading that never mixes depths).
Cache rows are addressed by slot; a row attends to ``slots[0..pos]``.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Sequence, Tuple

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(_build.build())
        dp = ctypes.POINTER(ctypes.c_double)
        fp = ctypes.POINTER(ctypes.c_float)
        ip = ctypes.POINTER(ctypes.c_int)
        _lib.orc_layer.argtypes = [ctypes.c_int] * 4 + [ctypes.c_double] * 3 + [fp] * 6 + [
            dp, ctypes.c_int, dp, dp, ip, ctypes.c_int]
        _lib.orc_logits.argtypes = [ctypes.c_int, ctypes.c_int, dp, fp, ctypes.c_double, fp, dp]
        _lib.orc_matvec.argtypes = [ctypes.c_int, ctypes.c_int, fp, dp, dp]
        _lib.orc_rmsnorm.argtypes = [ctypes.c_int, dp, fp, ctypes.c_double, dp]
        _lib.orc_rope.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, dp]
        _lib.orc_attend.argtypes = [ctypes.c_int] * 4 + [dp, dp, dp, ip, dp]
    return _lib


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _fp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


class LoopedModel:
    """P / B / C of a looped LM with slot-addressed per-(layer, depth) caches.

    ``weights``: dict of fp32 arrays from ``synthetic.make_weights`` (bf16
    models carry their bf16-rounded values).
    """

    def __init__(self, cfg, weights: Dict[str, np.ndarray], n_slots: int,
                 unwritten: float = 0.0):
        """``unwritten``: value of cache rows no position has written (NaN makes
        any read of a row that was never computed poison the result)."""
        self.cfg = cfg
        self.w = {k: np.ascontiguousarray(v, dtype=np.float32) for k, v in weights.items()}
        self.n_slots = n_slots
        self.unwritten = unwritten
        self.caches: Dict[Tuple[str, int], Tuple[np.ndarray, np.ndarray]] = {}
        self.lib = lib()

    # -- caches --------------------------------------------------------------
    def cache(self, layer: str, tag: int) -> Tuple[np.ndarray, np.ndarray]:
        key = (layer, tag)
        if key not in self.caches:
            d = self.cfg.d_model
            self.caches[key] = (np.full((self.n_slots, d), self.unwritten),
                                np.full((self.n_slots, d), self.unwritten))
        return self.caches[key]

    # -- one layer -----------------------------------------------------------
    def layer(self, name: str, tag: int, h: np.ndarray, pos: int, slots: Sequence[int],
              s: float) -> None:
        c = self.cfg
        assert len(slots) == pos + 1
        K, V = self.cache(name, tag)
        sl = np.ascontiguousarray(slots, dtype=np.int32)
        w = self.w
        self.lib.orc_layer(c.d_model, c.n_heads, c.head_dim, c.ffn, c.rms_eps, c.rope_theta, s,
                           _fp(w[f"{name}.g1"]), _fp(w[f"{name}.wqkv"]), _fp(w[f"{name}.wo"]),
                           _fp(w[f"{name}.g2"]), _fp(w[f"{name}.wgu"]), _fp(w[f"{name}.wd"]),
                           _dp(h), pos, _dp(K), _dp(V), _ip(sl), int(slots[-1]))

    # -- P, B, C (Eq. 1) -----------------------------------------------------
    def prelude(self, token: int, pos: int, slots: Sequence[int]) -> np.ndarray:
        """H^(0) = P(prefix): embedding row, then the prelude layers (scale 1)."""
        h = self.w["embed"][token].astype(np.float64)
        for i in range(self.cfg.n_prelude):
            self.layer(f"pre{i}", 0, h, pos, slots, 1.0)
        return h

    def iterate(self, h: np.ndarray, r: int, pos: int, slots: Sequence[int]) -> np.ndarray:
        """H^(r) = B(H^(r-1)): all shared layers with the depth-r caches, scale s."""
        h = h.copy()
        for i in range(self.cfg.n_core):
            self.layer(f"core{i}", r, h, pos, slots, self.cfg.resid_scale)
        return h

    def coda(self, h: np.ndarray, r: int, pos: int, slots: Sequence[int]) -> np.ndarray:
        hc = h.copy()
        for i in range(self.cfg.n_coda):
            self.layer(f"coda{i}", r, hc, pos, slots, 1.0)
        return hc

    def logits(self, hc: np.ndarray) -> np.ndarray:
        c = self.cfg
        z = np.empty(c.vocab)
        self.lib.orc_logits(c.d_model, c.vocab, _dp(hc), _fp(self.w["final_norm"]), c.rms_eps,
                            _fp(self.w["head"]), _dp(z))
        return z

    def readout(self, h: np.ndarray, r: int, pos: int, slots: Sequence[int]) -> np.ndarray:
        """Logits of C(H^(r)): coda layers (depth-r coda cache), final norm, LM head."""
        return self.logits(self.coda(h, r, pos, slots))
