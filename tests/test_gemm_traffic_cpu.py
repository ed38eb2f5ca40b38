"""Host logic behind the benchmark's roofline.traffic: the ncu CSV summary of
the weight-streaming GEMM's DRAM bytes (looped_transformer_self_b200/gemm_traffic.py).

A CSV in ncu's --csv layout (preamble lines, quoted header, one row per
(launch, metric), byte units that vary per row) with known values: the
summary gives each launch's read + write bytes in bytes, its algorithmic
bytes (weights + activation rows + fp32 result), their ratio, the per-launch
means, and the hash of the GEMM sources it was captured with."""
import csv

from looped_transformer_self_b200 import gemm_traffic as gt

HDR = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream",
       "Block Size", "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit",
       "Metric Value"]


def _write(path, launches):
    with open(path, "w", newline="") as f:
        f.write("==PROF== Connected to process 1 (python)\n")
        w = csv.writer(f, quoting=csv.QUOTE_ALL)
        w.writerow(HDR)
        for i, (rd, rd_u, wr, wr_u, us) in enumerate(launches):
            base = [str(i), "1", "python", "127.0.0.1", "void k_gemm<0, 16>(...)", "1", "7",
                    "(192, 1, 1)", "(148, 1, 1)", "0", "10.0", "Command line profiler metrics"]
            w.writerow(base + ["dram__bytes_read.sum", rd_u, f"{rd:,}"])
            w.writerow(base + ["dram__bytes_write.sum", wr_u, str(wr)])
            w.writerow(base + ["gpu__time_duration.sum", "usecond", str(us)])


def test_summary_of_known_launches(tmp_path):
    shapes = gt.shapes("huginn35")
    assert [s[0] for s in shapes] == ["qkv", "o", "gate_up", "down"]
    ncols = 16
    alg = [gt.algorithmic_bytes(n, k, ncols) for _, n, k in shapes]
    # reads of 1.01 x the algorithmic bytes in mixed units, small writes
    launches = [(int(alg[0] * 1.01), "byte", 1000, "byte", 30.0),
                (alg[1] * 1.01 / 1e6, "Mbyte", 2000, "byte", 10.0),
                (alg[2] * 1.01 / 1e9, "Gbyte", 3000, "byte", 60.0),
                (alg[3] * 1.01 / 1e3, "Kbyte", 4, "Kbyte", 35.0)]
    p = tmp_path / "traffic.csv"
    _write(p, [(round(r, 6) if u != "byte" else r, u, w, wu, us) for r, u, w, wu, us in launches])
    rec = gt.summarise(str(p), "huginn35", ncols)
    assert rec["model"] == "huginn35" and rec["ncols"] == ncols
    assert rec["source_sha256"] == gt.source_hash()
    writes = [1000, 2000, 3000, 4000]
    for o, a, wr in zip(rec["launches"], alg, writes):
        assert abs(o["algorithmic_bytes"] - a) < 1e-6 * a
        assert abs(o["dram_write"] - wr) < 1e-6 * max(wr, 1)
        assert abs(o["traffic_over_algorithmic"] - (1.01 + wr / a)) < 1e-5
    assert abs(rec["algorithmic_per_launch"] - sum(alg) / 4) < 1e-6 * sum(alg)
    assert abs(rec["traffic_per_launch"] - sum(o["traffic"] for o in rec["launches"]) / 4) < 1.0


def test_algorithmic_bytes_formula():
    # bf16 weights [n_out x k] + bf16 rows [ncols x k] + fp32 result [ncols x n_out]
    assert gt.algorithmic_bytes(128, 64, 16) == 2 * 128 * 64 + 2 * 16 * 64 + 4 * 16 * 128


def _bench():
    import importlib.util
    import os
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_bench_reports_traffic_only_for_a_matching_capture(tmp_path):
    import json
    bench = _bench()
    rec = {"model": "huginn35", "source_sha256": gt.source_hash(),
           "traffic_per_launch": 1.02e8, "algorithmic_per_launch": 1.0e8}
    p = tmp_path / "cap.json"
    p.write_text(json.dumps(rec))
    t, note = bench.gemm_traffic("huginn35", 2.0e8, str(p))
    assert abs(t - 2.04e8) < 1.0 and "1.0200" in note
    t, note = bench.gemm_traffic("ouro14", 2.0e8, str(p))
    assert t is None and "huginn35" in note
    p.write_text(json.dumps(dict(rec, source_sha256="0" * 64)))
    t, note = bench.gemm_traffic("huginn35", 2.0e8, str(p))
    assert t is None and "changed" in note
    t, note = bench.gemm_traffic("huginn35", 2.0e8, str(tmp_path / "absent.json"))
    assert t is None and note == "no capture"
    # the committed capture matches the committed GEMM sources and the default workload
    t, note = bench.gemm_traffic("huginn35", 1.0e8)
    assert t is not None and 0.9e8 < t < 1.2e8, note
