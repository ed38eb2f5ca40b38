"""CPU oracle for pipelined self-speculative decoding of looped Transformers.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call, link
or execute anything under ``oracle/``: only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` use it.  It shares no code with the
CUDA library; both take their inputs from the ``synthetic`` module.

It follows "LoopSpec: Pipelined Self-Speculative Decoding for Looped
Transformers" (liuzhao09.github.io/papers/loopspec.html):

  model.c / model.py   Eq. 1 (section 2.1): prelude P, shared block B looped R
                       times, coda/readout C; per-depth caches (Fig. 2); the
                       layer arithmetic in fp64.
  sampling.py          readout processing (temperature, top-p, normalisation;
                       section 2.1), the residual operator of Eq. 2, the
                       accept/resample rules of Eqs. 3-4 and the cascade of
                       section 2.3, Philox-4x32-10 and the exponential race.
  decode.py            prefill + first commit, full-depth autoregressive
                       decoding, and the pipelined speculative state machine of
                       sections 2.2-2.4 (proposals at d1 and d2, confidence gate
                       of Eq. 6, verify at R, prune / reroot, index-copy caches).
  depth.py             the depth-selection formula of Eq. 8 (section 2.4).

Every function is pinned by tests/test_oracle_*.py against facts the pages or
mathematics fix (see each test's docstring).
"""
