"""DRAM traffic of the weight-streaming GEMM on the shared-block shapes.

Runs lt_gemm_rows once on each of a model's four shared-block weight shapes
(QKV [3d x d], O [d x d], gate/up [2f x d], down [d x f]; bf16, random values)
with the decode step's row capacity, so a kernel profiler can read each
launch's DRAM bytes next to its algorithmic bytes (weights + activation rows +
fp32 result).  The matrices (0.8 GB for the Huginn-3.5B shape) exceed the
126 MB L2, so DRAM figures are not L2 hits.  Typical use (one GPU):

    ncu --clock-control none -k regex:k_gemm -c 4 \\
        --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum \\
        --csv --log-file traffic.csv \\
        python -m looped_transformer_self_b200.gemm_traffic --model huginn35

then `python -m looped_transformer_self_b200.gemm_traffic --summarise traffic.csv
--model huginn35` prints per-launch traffic and writes the record the
benchmark reads (profiles/gemm_traffic.json), stamped with a hash of the GEMM
sources.
"""
import argparse
import csv
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GEMM_SOURCES = ("gemm.cu", "gemm.cuh", "gemm_epi.cuh", "tc.cuh", "common.cuh")


def source_hash() -> str:
    """sha256 over the sources that make up the GEMM kernel."""
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, "looped_transformer_self_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def shapes(model: str):
    import synthetic as syn
    c = syn.MODELS[model]
    d, f = c.d_model, c.ffn
    return [("qkv", 3 * d, d), ("o", d, d), ("gate_up", 2 * f, d), ("down", d, f)]


def algorithmic_bytes(n_out: int, k: int, ncols: int) -> float:
    return 2.0 * n_out * k + 2.0 * ncols * k + 4.0 * ncols * n_out


def run(model: str, ncols: int) -> None:
    import torch
    from looped_transformer_self_b200.binding import gemm_rows
    g = torch.Generator().manual_seed(0)
    for name, n_out, k in shapes(model):
        w = torch.randn(n_out, k, generator=g).bfloat16().cuda()
        x = torch.randn(ncols, k, generator=g).bfloat16().cuda()
        y = gemm_rows(w, x)
        torch.cuda.synchronize()
        assert torch.isfinite(y).all(), name
        del w, x, y
    print(f"ran {len(shapes(model))} GEMM shapes of {model} with {ncols} rows")


def summarise(path: str, model: str, ncols: int) -> dict:
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    h = rows[hi]
    idc, mi, vi, ui = h.index("ID"), h.index("Metric Name"), h.index("Metric Value"), h.index("Metric Unit")
    per = {}
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6, "GB": 1e9,
             "nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "ns": 1e-3, "us": 1.0, "ms": 1e3}
    for r in rows[hi + 1:]:
        if len(r) <= vi:
            continue
        v = float(r[vi].replace(",", "")) * scale.get(r[ui], 1.0)
        per.setdefault(int(r[idc]), {})[r[mi]] = v
    launches = [per[k] for k in sorted(per)]
    out = []
    for (name, n_out, k), m in zip(shapes(model), launches):
        t = m["dram__bytes_read.sum"] + m["dram__bytes_write.sum"]
        a = algorithmic_bytes(n_out, k, ncols)
        out.append({"gemm": name, "n_out": n_out, "k": k, "algorithmic_bytes": a,
                    "dram_read": m["dram__bytes_read.sum"], "dram_write": m["dram__bytes_write.sum"],
                    "traffic": t, "traffic_over_algorithmic": t / a,
                    "duration_us_serialised": m.get("gpu__time_duration.sum")})
    rec = {"model": model, "ncols": ncols, "source_sha256": source_hash(), "launches": out,
           "traffic_per_launch": sum(o["traffic"] for o in out) / len(out),
           "algorithmic_per_launch": sum(o["algorithmic_bytes"] for o in out) / len(out)}
    return rec


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--model", default="huginn35")
    ap.add_argument("--ncols", type=int, default=16)
    ap.add_argument("--summarise", default=None, help="ncu csv of a run of this script")
    ap.add_argument("--out", default=os.path.join(ROOT, "profiles", "gemm_traffic.json"))
    args = ap.parse_args()
    if args.summarise:
        rec = summarise(args.summarise, args.model, args.ncols)
        print(json.dumps(rec, indent=1))
        json.dump(rec, open(args.out, "w"), indent=1)
    else:
        run(args.model, args.ncols)


if __name__ == "__main__":
    main()
