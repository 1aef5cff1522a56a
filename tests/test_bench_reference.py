"""The bench's reference arm (the CPU oracle timed on host cores) on the CPU:
one JSON line with the documented keys, on rank 0 only under torchrun."""
from __future__ import annotations

import json
import os
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["--impl", "reference", "--config", "c1_b16_g5_v32000_bf16", "--steps", "2", "--warmup",
        "3", "--ref-budget", "5"]


def _json_lines(out: str):
    return [json.loads(l) for l in out.splitlines() if l.startswith("{")]


def _check_line(d: dict, n_gpus: int):
    assert d["impl"] == "reference"
    assert d["metric"] and d["unit"] == "rows/s"
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == n_gpus and d["steps"] >= 1 and d["warmup"] >= 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["vs_baseline"] is None and d["data"] == "synthetic"
    assert d["config"]["workload"] == "c1_b16_g5_v32000_bf16"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["unit"] == d["unit"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # the rate is the workload's verified rows over the timed seconds
    assert abs(d["value"] * d["ms_per_step"] / 1e3 - 16 * 5) < 1e-6 * 16 * 5


def test_default_workload_is_the_largest_single_gpu_one():
    sys.path.insert(0, ROOT)
    import bench
    import workloads
    assert bench.DEFAULT_CONFIG == "c4_b256_g4_v151936_bf16"
    big = max(workloads.CONFIGS, key=lambda c: c.B * (2 * c.gamma + 1) * c.V)
    assert bench.DEFAULT_CONFIG == big.name
    # the oracle's timed sample of it is a bounded subset of whole sequences
    assert bench.oracle_batch(big) == 32 and bench.oracle_batch(workloads.get(1)) == 16


def test_reference_arm_single_process():
    r = subprocess.run([sys.executable, "bench.py", *ARGS], cwd=ROOT, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 1)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_reference_arm_under_torchrun_prints_once():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--gpus", "2", *ARGS]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    _check_line(lines[0], 2)
