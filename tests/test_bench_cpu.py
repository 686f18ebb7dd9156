"""The benchmark's reference arm (the CPU oracle on a bounded sample of the step) runs without a GPU
and prints the one JSON line the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_its_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
                        "--ref-seconds", "8"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["metric"] and d["unit"] == "TOPS" and d["steps"] == 1 and d["warmup"] == 1
    sys.path.insert(0, ROOT)
    import bench
    assert d["config"] == bench.bench_config(bench.WORKLOAD, 1)        # the same config as the GPU arm's line
    assert d["config"]["workload"] == "mlp_up_t16384_k8192_n28672"
    assert d["extrapolated"] is True and 0 < d["sample_fraction"]["tokens"] <= 1 and d["sample_seconds_per_step"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
