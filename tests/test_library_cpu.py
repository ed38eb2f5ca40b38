"""Host-side checks that need no GPU: the CUDA library builds for sm_100a,
loads, and exports every function include/looped_spec.h declares; the
product package refuses to run without its compiled library."""
import ctypes
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    txt = open(os.path.join(ROOT, "include", "looped_spec.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lt_[a-z0-9_]+)\s*\(", txt)))


def test_library_builds_and_exports_every_declared_symbol():
    from looped_transformer_self_b200 import build as B
    path = B.build()
    lib = ctypes.CDLL(path)
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(lib, n), n


def test_workspace_sizing_and_validation_without_gpu():
    import synthetic as syn
    from looped_transformer_self_b200 import binding as b
    L = b.lib()
    m = b.model_config_c(syn.MODELS["ouro14"])
    dc = b.DecodeConfigC(1, 2, 0.0, 1.0, 2, 16, 1600, 1024, 0, 0)
    n = ctypes.c_size_t()
    assert L.lt_workspace_bytes(ctypes.byref(m), ctypes.byref(dc), ctypes.byref(n)) == 0
    # KV pool: 24 layers x R=4 planes x slots x K/V x 2048 x bf16 dominates
    assert n.value > 24 * 4 * 1600 * 2 * 2048 * 2
    bad = b.DecodeConfigC(2, 2, 0.0, 1.0, 2, 16, 1600, 1024, 0, 0)  # d2 must exceed d1
    assert L.lt_workspace_bytes(ctypes.byref(m), ctypes.byref(bad), ctypes.byref(n)) == -2
    bad = b.DecodeConfigC(1, 2, 0.0, 1.0, 2, 12, 1600, 1024, 0, 0)  # capacity not a GEMM width
    assert L.lt_workspace_bytes(ctypes.byref(m), ctypes.byref(bad), ctypes.byref(n)) == -2
    m2 = b.model_config_c(syn.MODELS["ouro14"].replace(head_dim=100, n_heads=20, d_model=2000))
    assert L.lt_workspace_bytes(ctypes.byref(m2), ctypes.byref(dc), ctypes.byref(n)) == -2


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "looped_transformer_self_b200")
    for dp, _, fs in os.walk(pkg):
        for f in fs:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dp, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "liborc_model" not in src, f
