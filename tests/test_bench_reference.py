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


def test_stage_rooflines_arithmetic():
    """stage_rooflines: GB/s = bytes / time, the HBM fraction against the
    copy peak, TFLOP/s and both bf16 fractions only where the stage's
    arithmetic intensity is above the ridge, and stages with no work (fused
    into another) left out."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0}
    wk = {"route": {"bytes": 288_000_000, "flops": 34_000_000_000},
          "permute": {"bytes": 0, "flops": 0},
          "gate_up": {"bytes": 6_000_000_000, "flops": 6_600_000_000_000}}
    calls = {"route": 0.1, "permute": 0.003, "gate_up": 5.5}
    r = bench.stage_rooflines(wk, calls, pk)
    assert "permute" not in r
    assert abs(r["route"]["GB/s"] - 2880.0) < 0.1
    assert abs(r["route"]["frac_hbm"] - 2880.0 / 6650.0) < 1e-4
    assert "TFLOP/s" not in r["route"]  # 118 FLOP/B is below the ridge (239)
    tf = 6.6e12 / 5.5e-3 / 1e12
    assert abs(r["gate_up"]["TFLOP/s"] - tf) < 0.1
    assert abs(r["gate_up"]["frac_bf16_burst"] - tf / 1590.0) < 1e-4
    assert abs(r["gate_up"]["frac_bf16_sustained"] - tf / 1400.0) < 1e-4


def test_work_counts_follow_the_definitions():
    """bench.work: the router moves x, W_r, logits and routing; the expert
    GEMMs do 6 T k d f FLOPs; the permute reads x once and writes T k rows
    (or nothing where the GEMM gathers the rows itself); the combine reads
    T k rows and writes T rows."""
    sys.path.insert(0, ROOT)
    import bench
    from routing_dispatch_experts_b200 import workloads as W
    for cfg, w in W.WORKLOADS.items():
        wk = bench.work(w, w.T)
        b = 2 if w.dtype == "bf16" else 4
        R = w.T * w.k
        assert wk["route"]["flops"] == 2 * w.T * w.d * w.E
        assert wk["gate_up"]["flops"] + wk["down"]["flops"] == 6 * R * w.d * w.f
        assert wk["combine"]["bytes"] == R * w.d * b + w.T * w.d * b + 2 * R * 4
        gathered = w.dtype == "bf16" and w.T * w.d * b <= (96 << 20)
        assert wk["permute"]["bytes"] == (0 if gathered else w.T * w.d * b + R * w.d * b + R * 4)
