"""Host-side logic of bench.py (no GPU): the algorithmic byte and flop model
behind the roofline, the lookup of the profiled DRAM traffic, and the JSON
line of the reference arm (the oracle timed on the host cores)."""
import json
import os
import subprocess
import sys

import bench
from workloads import workload

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_fused_scan_model_at_the_2p7b_shape():
    w = workload("mamba2_2p7b_layer")
    m = bench.kernel_model(w, 35)["fused_scan"]
    b, T, H, P, N = 4, 4096, 80, 64, 128
    xy = 2 * b * T * H * P * 2              # X read and Y written, bf16
    bc = 2 * b * T * N * 2                  # B and C, one group
    la = b * T * H * 4
    fin = b * H * N * P * 4                 # final states
    nwork, _, ncuts = bench.fused_plan(w, 35)
    assert nwork == 147
    # the algorithmic bytes: the range states read at the cuts are a state spill, left out
    assert m["bytes"] == xy + bc + la + H * 4 + fin
    assert 355e6 < m["bytes"] < 365e6
    # per (b, tile, h): the masked quadratic term, the state read-out and update
    # (4 x 128 N P), and C B^T once per (b, tile, group)
    tiles = T // 128
    assert m["flops"] == b * tiles * (H * (128 * 129 * P + 4 * 128 * N * P) + 128 * 129 * N)
    # the same masked work as the primary count taken at block length 128 (54.0 GFLOP),
    # and the primary count at the workload's Q = 256 (65.0 GFLOP)
    assert abs(bench.algorithmic_flops(w, 128) - m["flops"]) < 1e-3 * m["flops"]
    assert abs(bench.algorithmic_flops(w) / 1e9 - 65.0) < 0.1 and abs(m["flops"] / 1e9 - 54.0) < 0.1


def test_profiled_traffic_belongs_to_the_current_source():
    v = bench.profiled_traffic("fused_scan")
    if v is None:
        return  # the summary was taken on another version of the kernel source
    w = workload("mamba2_2p7b_layer")
    alg = bench.kernel_model(w, 35)["fused_scan"]["bytes"]
    assert 0.8 * alg < v < 1.1 * alg  # no re-reads beyond what L2 absorbs
    assert bench.profiled_traffic("no_such_kernel") is None


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=240, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1 and line["warmup"] == 3
    assert line["metric"] and line["unit"] == "tokens·heads/s" and line["value"] > 0 and line["ms_per_step"] > 0
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["config"]["workload"] == "mamba2_2p7b_layer" and line["data"] == "synthetic"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
