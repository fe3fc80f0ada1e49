"""bench.py end to end on the GPU: the small workload's JSON line carries every
key the measurement contract asks for, with values that make sense."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_tiny_line():
    b = _run("--workload", "tiny", "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in b, k
    assert b["n_gpus"] == 1 and b["steps"] == 3 and b["warmup"] == 3
    assert b["value"] > 0 and b["ms_per_step"] > 0
    assert b["config"]["workload"].startswith("tiny")
    r = b["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["traffic"] is None            # the committed ncu summary covers the 480P workload only
    e = b["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert "rotate" in e["l2"]  # no flush inside the end-to-end region: caches rotate past L2
    assert b["gpu_launches"] == 2 * b["steps"]
    a = b["append"]
    assert a["bound"] == "alu" and 0 < a["frac"] < 1.5
    assert b["dense"]["ms"] > 0 and b["nonabsorbed"]["ms_total"] > 0
    assert set(b["dc_sweep"]) == {"64", "128", "192", "256"}
    assert b["splitkv"]["ms"] > 0 and b["splitkv"]["workspace_bytes"] == 0  # 5 key tiles: no split
    assert "chunk_480p" not in b and "other_workloads" not in b            # 480P run only


def test_bench_default_480p_line():
    # the default workload, short: the per-chunk schedules, the sustained loop and the
    # batch-8 / 1080P figures are in the line
    b = _run("--steps", "2", "--warmup", "3", "--no-cpu-baseline", "--chunk-replays", "2")
    assert b["config"]["workload"].startswith("480p")
    assert b["roofline"]["frac"] > 0.5
    c = b["chunk_480p"]
    for k in ("nonabsorbed", "nonabsorbed_reuse", "dense"):
        assert c[k]["ms_per_chunk"] > 0, k
    assert c["nonabsorbed_reuse"]["transient_kv_bytes"] < c["nonabsorbed"]["transient_kv_bytes"]
    s = c["sustained"]
    assert s["seconds"] >= 2.0 and s["attention_tflops"] > 0
    for name in ("480p_b8", "1080p"):
        o = b["other_workloads"][name]
        assert o["attention"]["ms"] > 0 and o["dense"]["ms"] > 0 and o["attention_splitkv"]["ms"] > 0
    assert b["other_workloads"]["1080p"]["attention_splitkv"]["workspace_bytes"] > 0


def test_bench_reference_arm_line():
    b = _run("--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0")
    assert b["impl"] == "reference"
    assert b["value"] > 0 and b["cpu_baseline"]["kind"] == "oracle"
    assert b["e2e"]["h2d_bytes_per_step"] == 0 and b["e2e"]["d2h_bytes_per_step"] == 0
    assert b["e2e"]["value"] == b["value"] and b["e2e"]["unit"] == b["unit"]
