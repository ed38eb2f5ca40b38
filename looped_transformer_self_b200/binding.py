"""ctypes binding of liblooped_spec.so (argument marshalling only).

Every call goes to the CUDA library; there is no other implementation.  If
the shared library is missing, the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblooped_spec.so")

LT_F32, LT_BF16 = 0, 1
ERRORS = {-1: "LT_ERR_ARG", -2: "LT_ERR_SHAPE", -3: "LT_ERR_CAPACITY", -4: "LT_ERR_CUDA",
          -5: "LT_ERR_DEVICE_CHECK", -6: "LT_ERR_STATE"}


class LoopedSpecError(RuntimeError):
    def __init__(self, code, msg=""):
        super().__init__(f"{ERRORS.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run __graft_entry__.build() "
                              "(or python looped_transformer_self_b200/build.py)")
        _lib = ctypes.CDLL(LIB_PATH)
        _declare(_lib)
    return _lib


_vp, _sz, _i = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int


def _declare(L):
    L.lt_gemm_scratch_bytes.argtypes = [_i, _i, _i, _i, ctypes.POINTER(_sz)]
    L.lt_gemm_rows.argtypes = [_i, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]
    for name in dir(L):
        pass


def check(code: int, what: str = "") -> None:
    if code != 0:
        raise LoopedSpecError(code, what)


def _ptr(t: torch.Tensor) -> int:
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def gemm_rows(w: torch.Tensor, x: torch.Tensor, scratch: torch.Tensor = None,
              stream=None) -> torch.Tensor:
    """Y[i][n] = sum_k x[i][k] w[n][k] through lt_gemm_rows (fp32 result)."""
    assert w.is_cuda and x.is_cuda and w.dtype == x.dtype
    dtype = LT_BF16 if w.dtype == torch.bfloat16 else LT_F32
    n_out, k = w.shape
    ncols = x.shape[0]
    need = _sz()
    check(lib().lt_gemm_scratch_bytes(dtype, n_out, k, ncols, ctypes.byref(need)))
    if scratch is None or scratch.numel() < need.value:
        scratch = torch.empty(need.value, dtype=torch.uint8, device=w.device)
    y = torch.empty(ncols, n_out, dtype=torch.float32, device=w.device)
    check(lib().lt_gemm_rows(dtype, _ptr(w), _ptr(x), _ptr(y), n_out, k, ncols, _ptr(scratch),
                             scratch.numel(), _stream(stream)), "lt_gemm_rows")
    return y
