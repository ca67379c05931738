"""The reference arm of bench.py (the CPU oracle), run as a user would on CPU.

Under torchrun only rank 0 runs and prints; the other ranks exit 0 at once.
Rank 0 prints one JSON line carrying the metric of the GPU arm, its own CPU
baseline description and an end-to-end entry with no host-device copies.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2")
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                          cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_other_ranks_exit_without_work():
    r = _run(1)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_rank0_prints_one_reference_line():
    r = _run(0)
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"].startswith("future-attn target TFLOP/s")
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["steps"] == 1 and d["config"]["workload"] == "qwen3_8b_16k"
    # The sample is one KV-head group (1/8 of the step's flops), the one the GPU arm's cpu_baseline times;
    # ms_per_step scales its time to a whole step.
    assert "KV head 0" in d["cpu_baseline"]["sample"] and "all 16384 positions" in d["cpu_baseline"]["sample"]
    assert abs(d["ms_per_step"] / d["sample_ms_per_step"] - 8.0) < 0.05
    sys.path.insert(0, ROOT)
    import bench
    from future_attention_targets_b200.workloads import WORKLOADS
    assert d["config"] == bench.workload_config(WORKLOADS["qwen3_8b_16k"], 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
