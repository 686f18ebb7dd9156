"""Benchmark of the smoothed W8A8 linear on B200.

One step is one pass of the whole path over one batch of synthetic, outlier-shaped input resident in
HBM, for the 70B-shaped MLP up-projection (T = 16384 tokens, K = 8192, N = 28672, RMSNorm-fed,
alpha 0.5, calibration 128 x 2048 tokens):
  1. abs-max of the RMSNorm output over the 262144 calibration tokens (4.3 GB read) and
  2. abs-max of the weight per input channel, both in one launch,
  3. smoothing factors s and the folded norm weight gamma / s,
  4. diag(s) W quantised to INT8 per output channel,
  5. fused RMSNorm(gamma / s) + per-token INT8 quantisation of the 16384 tokens,
  6. INT8 x INT8 -> INT32 GEMM with the per-token x per-channel dequant epilogue to bf16.
With N > 1 GPUs every rank runs the same step on its own tokens (weak scaling) and the calibration
abs-maxima are combined with an NCCL all-reduce(MAX) between steps 1-2 and 3 -- the path's only exchange.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       (N > 1: launch with torchrun, one process per GPU)
Prints one JSON line (rank 0). ``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_quantization_calib_b200 import synth  # noqa: E402
from post_quantization_calib_b200 import dist as sqdist  # noqa: E402

WORKLOAD = synth.workload("mlp_up_t16384_k8192_n28672")
METRIC = "W8A8 smoothed-linear INT8 TOPS & % of dense INT8 peak; quant kernel GB/s"
UNIT = "TOPS"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0     # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)
CPU_SAMPLE_SECONDS = 15.0   # target CPU work of the cpu_baseline sample


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def src_sha(name: str) -> str:
    with open(os.path.join(ROOT, "post_quantization_calib_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(stage: str, source: str, workload: str):
    """DRAM bytes per launch of a stage's kernel from a committed ncu summary, if the counters were
    taken on the current kernel source at this workload (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(f"{workload}:{stage}")
    if not d or d.get("source_sha") != src_sha(source):
        return None
    return d.get("bytes_per_launch")


def bench_config(w, world):
    """The `config` object of the benchmark line (shared by both arms)."""
    return {"workload": w.name, "T": w.T, "K": w.K, "N": w.group_N(0), "calib_rows": w.calib_rows,
            "alpha": w.alpha, "norm": w.norm, "parallelism": f"dp{world}",
            "l2": f"inputs larger than L2: each step reads the {2 * w.calib_rows * w.K / 1e9:.1f} GB calibration set"}


# ------------------------------------------------------------------------------------------------
# Clocks and throttle reasons, sampled while the GPU works (read-only NVML queries).

_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU every `period` seconds on a host thread,
    from before the warm-up to after the timed steps; the summary covers the samples taken inside the
    timed window (or, when that window is shorter than three samples, the whole GPU-busy run, and
    says so). Falls back to `nvidia-smi -lms` where NVML cannot be loaded."""

    def __init__(self, device_index: int, period: float = 0.01):
        self.period = period
        self.samples = []          # (t, sm_mhz, reason_bits, power_w)
        self.max_mhz = None
        self.window = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        self._smi = None
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            try:
                h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + str(props.uuid))
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nvml, self._h = pynvml, h
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
        except Exception:
            self._nvml = None
        self._index = device_index

    def _poll(self):
        nv, h = self._nvml, self._h
        while not self._stop.is_set():
            try:
                t = time.monotonic()
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                rs = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((t, sm, rs, pw))
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
            return
        fields = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                  "clocks_event_reasons.sw_power_cap")
        try:
            self._smi = subprocess.Popen(["nvidia-smi", f"--id={self._index}", f"--query-gpu={fields}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._smi_t0 = time.monotonic()
        except OSError:
            self._smi = None

    def mark_window(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        elif self._smi is not None:
            self._smi.terminate()
            try:
                out, _ = self._smi.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self._smi.kill()
                out, _ = self._smi.communicate()
            bits = (0x8, 0x40, 0x20, 0x4)
            for i, line in enumerate(out.strip().splitlines()):
                p = [x.strip() for x in line.split(",")]
                if len(p) < 7:
                    continue
                try:
                    sm, self.max_mhz, pw = float(p[0]), float(p[1]), float(p[2])
                except ValueError:
                    continue
                rs = sum(b for b, v in zip(bits, p[3:7]) if v.lower() == "active")
                self.samples.append((self._smi_t0 + 0.1 * i, sm, rs, pw))   # approximate times
        inside = [s for s in self.samples if self.window and self.window[0] <= s[0] <= self.window[1]]
        scope = "timed steps"
        use = inside
        if len(inside) < 3:
            use = self.samples
            scope = "warm-up, stage breakdown and timed steps (the timed steps alone are shorter than three samples)"
        reasons = sorted({n for s in use for b, n in _REASONS.items() if s[2] & b})
        sm = [s[1] for s in use]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(use), "samples_in_timed_steps": len(inside), "scope": scope,
                "power_w_max": max((s[3] for s in use), default=None),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ------------------------------------------------------------------------------------------------
# Algorithmic work of each stage (bytes that must move, or integer ops), per launch.

def stage_work(T, N, K, calib_rows):
    return {
        # the calibration rows and the weight rows read, gamma read, both maxima written
        "calib_absmax": {"bytes": 2 * calib_rows * K + 2 * N * K + 4 * K + 4 * K + 4 * K, "bound": "hbm"},
        "scales": {"bytes": 4 * K * 5, "bound": "hbm"},
        "weight_quant": {"bytes": 2 * N * K + N * K + 4 * K + 4 * N, "bound": "hbm"},
        "act_quant": {"bytes": 2 * T * K + T * K + 4 * K + 4 * T, "bound": "hbm"},
        "gemm": {"ops": 2 * T * N * K, "bytes": T * K + N * K + 2 * T * N + 4 * T + 4 * N, "bound": "tensor"},
    }


def row_warps(K: int) -> int:
    """Warps per row group of the row kernels for rows of K elements (one row per unit above 2048)."""
    nvec = K // 8
    return 1 if nvec <= 256 else 2 if nvec <= 512 else 4 if nvec <= 1024 else 8


def kernel_of(K: int):
    g = row_warps(K)
    return {"calib_absmax": (f"k_absmax_pair<{g},8,1,NORM>", "sq_rowwise.cu"), "scales": ("k_scales", "sq_rowwise.cu"),
            "weight_quant": (f"k_rows<{g},8,1,QUANT>", "sq_rowwise.cu"),
            "act_quant": (f"k_rows<{g},8,1,QUANT,NORM>", "sq_rowwise.cu"), "gemm": ("k_w8a8_linear<256>", "sq_gemm.cu")}


LAUNCHES = {"calib_absmax": 2, "scales": 1, "weight_quant": 1, "act_quant": 1, "gemm": 1}


# ------------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reported CPU baseline and the reference arm).

def h16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_stage_seconds(w, f: float):
    """Seconds the oracle would take for every stage of one full step, each measured on a sample of
    about a fraction f of its rows and scaled linearly: the calibration rows (abs-max), the weight's
    output channels (weight abs-max, weight quantisation), the tokens (activation quantisation) and
    both for the GEMM (its time scales with tokens x channels). Returns (per-stage seconds, sample
    text, measured seconds of the sample, the fractions used)."""
    import oracle as orc
    T, K, N = w.T, w.K, w.group_N(0)
    rc = max(64, min(w.calib_rows, int(round(w.calib_rows * f))))
    rt = max(16, min(T, int(round(T * f))))
    rn = max(16, min(N, int(round(N * f))))
    ch = synth.outlier_channels(K, w.outliers, synth.seed_for(w.index, "outliers", 0))
    g = synth.norm_gamma(K, synth.seed_for(w.index, "gamma", 0)).numpy() if w.norm else None
    w16 = h16(synth.normal_weight(rn, K, synth.seed_for(w.index, "w", 0)))
    x16 = h16(synth.outlier_tokens(rt, K, ch, synth.seed_for(w.index, "x", 0)))
    c16 = h16(next(synth.calibration_chunks(w, ch, "cpu", rows=rc, chunk=rc)))
    t, meas = {}, 0.0

    def timed(fn):
        nonlocal meas
        t0 = time.perf_counter()
        out = fn()
        dt = time.perf_counter() - t0
        meas += dt
        return out, dt

    amax, dt = timed(lambda: orc.calibrate_absmax(c16, norm_gamma=g, eps=w.eps))
    t["calib_absmax"] = dt * (w.calib_rows / rc)
    aw, dt = timed(lambda: orc.calibrate_absmax(w16))
    t["weight_absmax"] = dt * (N / rn)
    (s, fold), dt = timed(lambda: orc.compute_scales(amax, aw, w.alpha, g))
    t["scales"] = dt
    (wq, ws), dt = timed(lambda: orc.smooth_quantize_weight(w16, s))
    t["weight_quant"] = dt * (N / rn)
    (xq, xs), dt = timed(lambda: orc.rmsnorm_smooth_quant(x16, fold, eps=w.eps, apply_norm=w.norm))
    t["act_quant"] = dt * (T / rt)
    _, dt = timed(lambda: orc.w8a8_linear(xq, xs, wq, ws))
    t["gemm"] = dt * (T / rt) * (N / rn)
    sample = (f"{rc} of {w.calib_rows} calibration rows, {rn} of {N} weight rows, {rt} of {T} tokens "
              f"(GEMM {rt} x {rn} x {K}); each stage's time scaled linearly to the full step (the GEMM by "
              f"tokens x channels)")
    return t, sample, meas, {"calib_rows": rc / w.calib_rows, "weight_rows": rn / N, "tokens": rt / T}


def oracle_fraction(w, seconds: float) -> float:
    """Sample fraction whose oracle run takes about `seconds`, from a small probe (time ~ a f + b f^2:
    the GEMM term grows with tokens x channels)."""
    f0 = 1.0 / 512
    t, _, _, _ = oracle_stage_seconds(w, f0)
    lin = sum(v for k, v in t.items() if k not in ("gemm", "scales")) * f0
    quad = t["gemm"] * f0 * f0
    a, b = lin / f0, quad / (f0 * f0)
    if b <= 0:
        return min(1.0, seconds / max(a, 1e-9))
    f = (-a + (a * a + 4 * b * seconds) ** 0.5) / (2 * b)
    return max(f0, min(1.0, f))


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def reference_arm(args, rank, world):
    if rank != 0:
        return 0
    import oracle as orc
    cores = cpu_cores()
    orc.set_threads(cores)
    w = WORKLOAD
    # each step is a bounded sample, sized so that warm-up + timed steps end in about two minutes
    per_step = args.ref_seconds / max(1, args.steps + args.warmup)
    frac = oracle_fraction(w, per_step)
    for _ in range(args.warmup):
        oracle_stage_seconds(w, frac)
    steps, meas, sample, fr = [], [], "", {}
    for _ in range(args.steps):
        t, sample, m, fr = oracle_stage_seconds(w, frac)
        steps.append(sum(t.values()))
        meas.append(m)
    step = sum(steps) / len(steps)
    value = w.linear_ops() / step / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": bench_config(w, world),
        "extrapolated": True, "sample_fraction": fr, "sample_seconds_per_step": sum(meas) / len(meas),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
                         "threads": f"GEMM on {cores} OpenMP threads; the other stages run on one thread"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# GPU arm.

def main_gpu(args, rank, local_rank, world):
    import torch.distributed as dist
    from post_quantization_calib_b200 import build as sqbuild
    sqbuild.build()
    from post_quantization_calib_b200 import sq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    w = WORKLOAD
    T, K, N = w.T, w.K, w.group_N(0)
    d = synth.group_inputs(w, 0, dev, rank=rank)
    gamma, W, X = d["gamma"], d["weight"], d["x"]
    calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], dev, rank=rank)))   # resident in HBM
    amax = torch.empty(K, dtype=torch.float32, device=dev)
    aw = torch.empty(K, dtype=torch.float32, device=dev)
    s = torch.empty(K, dtype=torch.float32, device=dev)
    fold = torch.empty(K, dtype=torch.float32, device=dev)
    wq = torch.empty(N, K, dtype=torch.int8, device=dev)
    ws = torch.empty(N, dtype=torch.float32, device=dev)
    xq = torch.empty(T, K, dtype=torch.int8, device=dev)
    xs = torch.empty(T, dtype=torch.float32, device=dev)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)
    names = list(LAUNCHES)

    # ev: events recorded at the stage boundaries listed in `at` (None: all). bufs: the step's
    # (calibration set, weight, tokens, output) buffers (default: the resident ones).
    def step(ev=None, at=None, bufs=None):
        c_in, w_in, x_in, y_out = bufs if bufs is not None else (calib, W, X, y)

        def mark(i):
            if ev is not None and (at is None or i in at):
                ev[i].record(stream)
        mark(0)
        # S1 + S2: the calibration maxima (of the RMSNorm output) and the weight maxima, one launch
        sq.sq_calibrate_absmax_pair(c_in, w_in, norm_gamma=gamma, eps=w.eps, amax=amax, amax_w=aw,
                                    accumulate=False, stream=stream)
        if world > 1:
            sqdist.allreduce_max_(amax)         # every rank's calibration rows: the global maxima
        mark(1)
        sq.sq_compute_scales(amax, aw, w.alpha, gamma=gamma, s=s, fold=fold, stream=stream)
        mark(2)
        sq.sq_smooth_quantize_weight(w_in, s, wq=wq, w_scale=ws, stream=stream)
        mark(3)
        sq.sq_rmsnorm_smooth_quant(x_in, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs, stream=stream)
        mark(4)
        sq.sq_w8a8_linear(xq, xs, wq, ws, y=y_out, stream=stream)
        mark(5)

    def online(x_in, y_out):
        """The online path alone: per-token quantisation of the tokens, then the GEMM."""
        sq.sq_rmsnorm_smooth_quant(x_in, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs, stream=stream)
        sq.sq_w8a8_linear(xq, xs, wq, ws, y=y_out, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(max(3, args.warmup)):
        step()
    st = sq.sq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sq.sq_status_string(st)} after warm-up")

    # Stage breakdown: a separate, untimed pass with an event at every stage boundary. An event between
    # two kernels stops the second from starting early (dependent launch), so the timed steps below
    # record events only around the dominant stage.
    nb = max(3, min(args.steps, 100))
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(nb)]
    for i in range(nb):
        step(bevs[i])
    torch.cuda.synchronize()
    stage_ms = {n: 0.0 for n in names}
    for e in bevs:
        for j, n in enumerate(names):
            stage_ms[n] += e[j].elapsed_time(e[j + 1])
    stage_ms = {n: v / nb for n, v in stage_ms.items()}
    dom_i = max(range(len(names)), key=lambda j: stage_ms[names[j]])

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    h0 = time.monotonic()
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i], at=(dom_i, dom_i + 1))
    t_end.record(stream)
    torch.cuda.synchronize()
    h1 = time.monotonic()
    barrier()
    clocks.mark_window(h0, h1)
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    st = sq.sq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sq.sq_status_string(st)} after the timed steps")
    # the dominant stage's own time, live in the timed region
    stage_ms[names[dom_i]] = sum(e[dom_i].elapsed_time(e[dom_i + 1]) for e in evs) / args.steps

    t_max = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
    elapsed_ms = float(t_max.item())
    ms_per_step = elapsed_ms / args.steps
    value = world * w.linear_ops() * args.steps / (elapsed_ms * 1e-3) / 1e12

    # ---- end to end through the C ABI with host buffers. Two measurements:
    #   e2e         the whole step: the calibration set, the weight and the tokens are copied in from
    #               pinned host memory every step, y is copied back;
    #   e2e_online  the online path only (weights, scales and fold resident, as a served layer keeps
    #               them): the tokens in, per-token quantisation and the GEMM, y back.
    # Consecutive steps are pipelined as a user streaming batches would: two sets of device buffers,
    # host-to-device copies on one stream, device-to-host copies on another (separate copy engines),
    # the library calls on the compute stream. A step's copy into a buffer set waits until the step
    # two earlier has finished reading it; a step's output waits until its buffer's previous copy to
    # the host is done.
    e2e_steps = 0 if args.no_e2e else max(2, min(args.steps, 20))
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)

    def pipelined(n_steps, sets, host_in, y_hosts, run):
        """ms per step of `run(set)` over n_steps pipelined steps (see above)."""
        done_reading = [None, None]
        done_writing = [None, None]

        def one(i):
            k = i % 2
            dev_in, y_out = sets[k]
            with torch.cuda.stream(h2d_stream):
                if done_reading[k] is not None:
                    h2d_stream.wait_event(done_reading[k])
                for dst, src in zip(dev_in, host_in):
                    dst.copy_(src, non_blocking=True)
                loaded = torch.cuda.Event()
                loaded.record(h2d_stream)
            stream.wait_event(loaded)
            if done_writing[k] is not None:
                stream.wait_event(done_writing[k])
            run(dev_in, y_out)
            computed = torch.cuda.Event()
            computed.record(stream)
            done_reading[k] = computed
            with torch.cuda.stream(d2h_stream):
                d2h_stream.wait_event(computed)
                y_hosts[k].copy_(y_out, non_blocking=True)
                written = torch.cuda.Event()
                written.record(d2h_stream)
            done_writing[k] = written

        for i in range(2):
            one(i)
        barrier()
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        h2d_stream.wait_stream(stream)
        d2h_stream.wait_stream(stream)
        for i in range(n_steps):
            one(i)
        stream.wait_stream(d2h_stream)
        stream.wait_stream(h2d_stream)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n_steps

    e2e_ms = e2e_on_ms = float("nan")
    h2d = d2h = h2d_on = 0
    if e2e_steps:
        y_ref = y.cpu()
        y_hs = [torch.empty(T, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        X_h = X.cpu().pin_memory()
        # online path first (the smaller host buffers), then the whole step
        on_sets = [((X,), y), ((torch.empty_like(X),), torch.empty_like(y))]
        e2e_on_ms = pipelined(max(2, min(args.steps, 50)), on_sets, (X_h,), y_hs, lambda di, yo: online(di[0], yo))
        if not torch.equal(y_hs[1], y_ref) or not torch.equal(y_hs[0], y_ref):
            raise RuntimeError("online end-to-end output differs from the device-resident step's output")
        h2d_on = X.numel() * 2
        del on_sets
        calib_h, W_h = calib.cpu().pin_memory(), W.cpu().pin_memory()
        sets = [((calib, W, X), y),
                ((torch.empty_like(calib), torch.empty_like(W), torch.empty_like(X)), torch.empty_like(y))]
        e2e_ms = pipelined(e2e_steps, sets, (calib_h, W_h, X_h), y_hs,
                           lambda di, yo: step(bufs=(di[0], di[1], di[2], yo)))
        if not torch.equal(y_hs[(e2e_steps - 1) % 2], y_ref):
            raise RuntimeError("end-to-end output differs from the device-resident step's output")
        h2d = (calib.numel() + W.numel() + X.numel()) * 2
        d2h = y.numel() * 2
        del sets, calib_h, W_h
    te = torch.tensor([e2e_ms, e2e_on_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_ms, e2e_on_ms = float(te[0].item()), float(te[1].item())

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    int8_burst = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    int8_sust = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])) * INT8_PER_BF16
    work = stage_work(T, N, K, w.calib_rows)
    stages = {}
    for n in names:
        ms = stage_ms[n]
        wk = work[n]
        ent = {"ms": ms, "launches": LAUNCHES[n], "timed": "live" if n == names[dom_i] else "breakdown pass"}
        if wk["bound"] == "tensor":
            ent["tops"] = wk["ops"] / (ms * 1e-3) / 1e12
            ent["frac_of_int8_sustained"] = ent["tops"] / int8_sust
            ent["frac_of_int8_burst"] = ent["tops"] / int8_burst
        ent["gbs"] = wk["bytes"] / (ms * 1e-3) / 1e9
        ent["frac_of_hbm"] = ent["gbs"] / hbm
        stages[n] = ent
    dom = names[dom_i]
    kern, srcfile = kernel_of(K)[dom]
    if work[dom]["bound"] == "tensor":
        # the GEMM is timed inside a seconds-long loop of steps: the sustained (power-capped) reference
        roof = {"bound": "tensor", "achieved": stages[dom]["tops"], "peak": int8_sust, "unit": "TOPS",
                "frac": stages[dom]["tops"] / int8_sust, "frac_of_burst": stages[dom]["tops"] / int8_burst}
        peak_note = (f"int8 peak = {src} sustained bf16 {peaks.get('bf16_tflops_sustained')} TFLOP/s x "
                     f"{INT8_PER_BF16:g} (nominal int8/bf16 ratio); frac_of_burst against the {src} burst "
                     f"{peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16:g}")
    else:
        roof = {"bound": "hbm", "achieved": stages[dom]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": stages[dom]["gbs"] / hbm}
        peak_note = f"HBM peak = {src} copy bandwidth"
    roof["traffic"] = recorded_traffic(dom, srcfile, w.name)
    roof["kernel"] = kern
    roof["stage"] = dom
    roof["peak_source"] = peak_note

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle as orc
        cores = cpu_cores()
        orc.set_threads(cores)
        frac = oracle_fraction(w, CPU_SAMPLE_SECONDS)
        st_s, sample, meas, fr = oracle_stage_seconds(w, frac)
        secs = sum(st_s.values())
        cpu = {"value": w.linear_ops() / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": sample, "sample_seconds": meas, "sample_fraction": fr, "extrapolated": True,
               "threads": f"GEMM on {cores} OpenMP threads; the other stages (act_quant included) on one thread",
               "stage_seconds": st_s}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": bench_config(w, world),
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": world * w.linear_ops() / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "what": "whole step: calibration set, weight and tokens copied in, y copied out"},
        "e2e_online": {"value": world * w.linear_ops() / (e2e_on_ms * 1e-3) / 1e12, "unit": UNIT,
                       "h2d_bytes_per_step": h2d_on, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_on_ms,
                       "what": "online path: tokens copied in, per-token quantisation and GEMM, y copied out; "
                               "weights, scales and fold resident"},
        "gpu_launches": sum(LAUNCHES.values()) * args.steps,
        "clocks": clk,
        "stages": stages,
        "stages_note": (f"the dominant stage is timed in the timed steps with events around it only; the others come "
                        f"from a separate pass of {nb} steps with an event at every stage boundary (those events "
                        f"block the dependent launch, so they stay out of the timed steps)"),
        "gemm_tops": stages["gemm"]["tops"],
        "gemm_frac_of_int8_sustained": stages["gemm"]["frac_of_int8_sustained"],
        "gemm_frac_of_int8_burst": stages["gemm"]["frac_of_int8_burst"],
        "quant_kernel_gbs": stages["act_quant"]["gbs"],
        "online_ms_per_step": stage_ms["act_quant"] + stage_ms["gemm"],
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed CPU oracle sample")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurements")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: CPU seconds for all its warm-up and timed steps together")
    args = ap.parse_args()
    rank, local_rank, world = sqdist.env_rank()
    if world != args.gpus and world == 1 and args.gpus > 1:
        print(f"--gpus {args.gpus} needs torchrun with {args.gpus} processes", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    return main_gpu(args, rank, local_rank, world)


if __name__ == "__main__":
    sys.exit(main())
