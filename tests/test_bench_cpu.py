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


def test_reference_arm_under_two_ranks():
    """Launched as the multi-GPU runs are (torchrun, two processes on 127.0.0.1): rank 0 alone times the
    oracle and prints the line (n_gpus 2, parallelism dp2); the other rank exits 0 without work."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "1", "--ref-seconds", "4"],
                       cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["config"]["parallelism"] == "dp2" and d["value"] > 0


def test_clock_summary_keeps_to_the_timed_window_and_names_reasons():
    """The clock record summarises the samples inside the timed steps (falling back to the whole run,
    and saying so, when that window holds fewer than three) and names every active slowdown reason."""
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c._thread, c._smi, c._nvml, c.max_mhz = None, None, object(), 1965.0
    c.samples = [(0.0, 1965.0, 0, 300.0), (1.0, 1500.0, 0x4, 1000.0), (1.1, 1520.0, 0x4, 990.0),
                 (1.2, 1480.0, 0x4 | 0x40, 1001.0), (5.0, 1900.0, 0, 400.0)]
    c.window = (0.9, 1.3)
    r = c.stop()
    assert r["samples"] == r["samples_in_timed_steps"] == 3 and r["scope"] == "timed steps"
    assert r["sm_mhz"] == 1500.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"] and r["power_w_max"] == 1001.0
    c.window = (4.0, 6.0)                    # one sample inside: the whole run is summarised instead
    r = c.stop()
    assert r["samples"] == 5 and r["samples_in_timed_steps"] == 1 and r["scope"] != "timed steps"


def test_oracle_sample_fraction_and_stage_scaling():
    """The CPU baseline's sample: the fraction solves a f + b f^2 = seconds for the probe's linear and
    GEMM terms, and every stage time is scaled to the full step (the GEMM by tokens x channels)."""
    sys.path.insert(0, ROOT)
    import bench
    w = bench.synth.workload("single_linear_t256_k1024_n1024")
    t, sample, meas, fr = bench.oracle_stage_seconds(w, 0.25)
    assert set(t) == {"calib_absmax", "weight_absmax", "scales", "weight_quant", "act_quant", "gemm"}
    assert all(v >= 0 for v in t.values()) and meas > 0 and "scaled" in sample
    assert 0 < fr["tokens"] <= 1 and 0 < fr["weight_rows"] <= 1 and 0 < fr["calib_rows"] <= 1
    f = bench.oracle_fraction(w, 0.05)
    assert 1.0 / 512 <= f <= 1.0
