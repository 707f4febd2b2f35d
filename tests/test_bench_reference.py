"""`bench.py --impl reference` (the oracle timed on the host cores) prints
one JSON line with the keys the benchmark contract asks of that arm, on the
same metric, unit and workload description as the measured arm.  No GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_default_workload_is_the_largest():
    """With no flags the benchmark measures the largest single-GPU workload."""
    sys.path.insert(0, ROOT)
    import bench
    from routing_dispatch_experts_b200 import workloads as W
    big = max(W.WORKLOADS.values(), key=lambda w: 6 * w.T * w.k * w.d * w.f)
    assert bench.DEFAULT_CONFIG == big.cfg == 5


def test_reference_arm_json_line():
    # the fine-grained workload keeps this CPU test short (its expert weights
    # are small); the arm runs the same code for every workload
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1",
                          "--warmup", "3", "--config", "2"], cwd=ROOT, capture_output=True,
                         text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config"):
        assert key in j, key
    assert j["metric"] == "MoE-layer fwd routed tokens/s" and j["unit"] == "tokens/s"
    assert j["higher_is_better"] is True and j["value"] > 0
    assert j["steps"] == 1 and j["warmup"] >= 3 and j["n_gpus"] == 1
    assert j["dtype"] == "f64" and j["data"] == "synthetic"
    assert "workload" in j["config"] and "T=16384" in j["config"]["workload"]
    cb = j["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == j["value"] and cb["cores"] >= 1
    assert cb["unit"] == j["unit"] and cb["sample"]
    e2e = j["e2e"]
    assert e2e == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}
