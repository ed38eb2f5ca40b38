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


def test_copy_settings_are_validated_without_gpu():
    import synthetic as syn
    from looped_transformer_self_b200 import binding as b
    L = b.lib()
    m = b.model_config_c(syn.MODELS["ouro14"])
    n = ctypes.c_size_t()

    def dc(*copy):
        return b.DecodeConfigC(1, 2, 0.0, 1.0, 2, 32, 1600, 1024, 0, 0, *copy)

    assert L.lt_workspace_bytes(ctypes.byref(m), ctypes.byref(dc(4, 16, 64, 7, 0.02)), ctypes.byref(n)) == 0
    for bad in [(4, 33, 64, 7, 0.02),   # longer than the 32-token limit
                (4, 0, 64, 7, 0.02),    # empty proposals
                (8, 16, 4, 7, 0.02),    # match cap below k
                (4, 16, 64, -1, 0.02),  # negative reserve
                (4, 16, 64, 7, -0.5),   # negative threshold
                (-1, 16, 64, 7, 0.0)]:
        assert L.lt_workspace_bytes(ctypes.byref(m), ctypes.byref(dc(*bad)), ctypes.byref(n)) == -2, bad


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference times the CPU oracle and prints one JSON line
    with the contract's keys (small model so it ends in seconds)."""
    import json
    import subprocess
    import sys
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--model", "tiny", "--steps", "1", "--warmup", "3"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "cpu_baseline", "e2e", "config"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["config"]["workload"].startswith("tiny")
    assert line["e2e"]["h2d_bytes_per_step"] == 0
