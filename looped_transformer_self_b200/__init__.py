"""B200 (sm_100a) library for pipelined self-speculative decoding of looped
Transformers ("LoopSpec", liuzhao09.github.io/papers/loopspec.html).

The compute path lives in ``liblooped_spec.so`` (CUDA C++, C ABI declared in
include/looped_spec.h).  ``binding`` is a thin ctypes layer with the same
names: argument marshalling only.  PyTorch supplies device memory and streams.
"""
from .binding import lib, LoopedSpecError  # noqa: F401
