"""Benchmark of the smoothed W8A8 linear on B200.

One step is one pass of the whole path over one batch of synthetic, outlier-shaped input resident in
HBM, for the Qwen3-8B-shaped query projection (T = 8192 tokens, K = N = 4096, RMSNorm-fed, alpha 0.5):
  1. abs-max of the RMSNorm output over 128 x 512 calibration tokens (537 MB read) and
  2. abs-max of the weight per input channel, both in one launch,
  3. smoothing factors s and the folded norm weight gamma / s,
  4. diag(s) W quantised to INT8 per output channel,
  5. fused RMSNorm(gamma / s) + per-token INT8 quantisation of the 8192 tokens,
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
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_quantization_calib_b200 import synth  # noqa: E402
from post_quantization_calib_b200 import dist as sqdist  # noqa: E402

WORKLOAD = synth.workload("qproj_t8192_k4096_n4096")
METRIC = "W8A8 smoothed-linear INT8 TOPS & % of dense INT8 peak; quant kernel GB/s"
UNIT = "TOPS"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0     # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)


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


def recorded_traffic(stage: str, source: str):
    """DRAM bytes per launch of a stage's kernel from a committed ncu summary, if the counters were
    taken on the current kernel source (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(stage)
    if not d or d.get("source_sha") != src_sha(source):
        return None
    return d.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# Algorithmic work of each stage (bytes that must move, or integer ops), per launch.

def stage_work(w, T, N, K, calib_rows):
    return {
        # the calibration rows and the weight rows read, gamma read, both maxima written
        "calib_absmax": {"bytes": 2 * calib_rows * K + 2 * N * K + 4 * K + 4 * K + 4 * K, "bound": "hbm"},
        "scales": {"bytes": 4 * K * 5, "bound": "hbm"},
        "weight_quant": {"bytes": 2 * N * K + N * K + 4 * K + 4 * N, "bound": "hbm"},
        "act_quant": {"bytes": 2 * T * K + T * K + 4 * K + 4 * T, "bound": "hbm"},
        "gemm": {"ops": 2 * T * N * K, "bytes": T * K + N * K + 2 * T * N + 4 * T + 4 * N, "bound": "tensor"},
    }


KERNEL_OF = {"calib_absmax": ("k_absmax_pair<2,8,1,NORM>", "sq_rowwise.cu"),
             "scales": ("k_scales", "sq_rowwise.cu"), "weight_quant": ("k_rows<2,8,1,QUANT>", "sq_rowwise.cu"),
             "act_quant": ("k_rows<2,8,1,QUANT,NORM>", "sq_rowwise.cu"), "gemm": ("k_w8a8_linear<256>", "sq_gemm.cu")}
LAUNCHES = {"calib_absmax": 2, "scales": 1, "weight_quant": 1, "act_quant": 1, "gemm": 1}


# ------------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample (the reported CPU baseline and the reference arm).

def h16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_step_seconds(w, frac: float):
    """Seconds for the oracle to run one full step, measured on a 1/frac-sized sample and scaled
    linearly (every stage is linear in the rows it processes). Returns (seconds, sample text)."""
    import oracle as orc
    T, K, N = w.T, w.K, w.group_N(0)
    rc = max(64, int(w.calib_rows * frac))
    rt = max(16, int(T * frac))
    d = synth.group_inputs(w, 0, "cpu", T=rt)
    calib = next(synth.calibration_chunks(w, d["channels"], "cpu", rows=rc, chunk=rc))
    g = d["gamma"].numpy() if d["gamma"] is not None else None
    c16, w16, x16 = h16(calib), h16(d["weight"]), h16(d["x"])
    t = {}
    t0 = time.perf_counter()
    amax = orc.calibrate_absmax(c16, norm_gamma=g, eps=w.eps)
    t["calib_absmax"] = (time.perf_counter() - t0) * (w.calib_rows / rc)
    t0 = time.perf_counter()
    aw = orc.calibrate_absmax(w16)
    t["weight_absmax"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    s, fold = orc.compute_scales(amax, aw, w.alpha, g)
    t["scales"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    wq, ws = orc.smooth_quantize_weight(w16, s)
    t["weight_quant"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    xq, xs = orc.rmsnorm_smooth_quant(x16, fold, eps=w.eps, apply_norm=w.norm)
    t["act_quant"] = (time.perf_counter() - t0) * (T / rt)
    t0 = time.perf_counter()
    orc.w8a8_linear(xq, xs, wq, ws)
    t["gemm"] = (time.perf_counter() - t0) * (T / rt)
    sample = (f"{rc} of {w.calib_rows} calibration rows, {rt} of {T} tokens (quantisation and GEMM rows), "
              f"full weight; times scaled linearly to the full step")
    return sum(t.values()), sample, t


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
    # size each step so that warm-up + timed steps finish in about two minutes
    probe, _, _ = oracle_step_seconds(w, 1.0 / 256)
    full = probe
    per_step_budget = 120.0 / max(1, args.steps + args.warmup)
    frac = min(1.0 / 16, max(1.0 / 2048, per_step_budget / max(full, 1e-9)))
    for _ in range(args.warmup):
        oracle_step_seconds(w, frac)
    secs, sample = [], ""
    for _ in range(args.steps):
        s, sample, _ = oracle_step_seconds(w, frac)
        secs.append(s)
    step = sum(secs) / len(secs)
    value = w.linear_ops() / step / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "K": w.K, "N": w.group_N(0), "calib_rows": w.calib_rows,
                   "alpha": w.alpha, "norm": w.norm},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
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
    calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], dev, rank=rank)))   # [65536, 4096] resident
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

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    st = sq.sq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sq.sq_status_string(st)} after warm-up")

    # Stage breakdown: a separate, untimed pass with an event at every stage boundary. An event between
    # two kernels stops the second from starting early (dependent launch) and cost ~20 us per step, so
    # the timed steps below record events only around the dominant stage.
    nb = max(3, min(args.steps, 200))
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

    clocks = ClockSampler(local_rank)
    clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i], at=(dom_i, dom_i + 1))
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    st = sq.sq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sq.sq_status_string(st)} after the timed steps")
    # the dominant stage's own time, live in the timed region
    stage_ms_breakdown = dict(stage_ms)
    stage_ms[names[dom_i]] = sum(e[dom_i].elapsed_time(e[dom_i + 1]) for e in evs) / args.steps

    t_max = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_max, op=dist.ReduceOp.MAX)
    elapsed_ms = float(t_max.item())
    ms_per_step = elapsed_ms / args.steps
    value = world * w.linear_ops() * args.steps / (elapsed_ms * 1e-3) / 1e12

    # ---- end to end through the C ABI with host buffers: every step copies its inputs from pinned
    # host memory and its output y back. Consecutive steps are pipelined as a user streaming batches
    # would: two sets of device buffers, host-to-device copies on one stream, device-to-host copies on
    # another (the two directions use separate copy engines), the library calls on the compute stream.
    # A step's copy into a buffer set waits until the step two earlier has finished reading it; a
    # step's output waits until its buffer's previous copy to the host is done.
    e2e_steps = 0 if args.no_e2e else max(2, min(args.steps, 20))
    pin = (lambda t: t.cpu().pin_memory()) if e2e_steps else (lambda t: t.cpu()[:0])
    calib_h, W_h, X_h = pin(calib), pin(W), pin(X)
    if e2e_steps:
        sets = [(calib, W, X, y), (torch.empty_like(calib), torch.empty_like(W), torch.empty_like(X), torch.empty_like(y))]
        y_hs = [torch.empty(T, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d_stream = torch.cuda.Stream(dev)
    d2h_stream = torch.cuda.Stream(dev)
    done_reading = [None, None]    # per buffer set: the compute of its last step has finished
    done_writing = [None, None]    # per buffer set: the copy of its last output to the host has finished

    def e2e_step(i):
        k = i % 2
        c_in, w_in, x_in, y_out = sets[k]
        with torch.cuda.stream(h2d_stream):
            if done_reading[k] is not None:
                h2d_stream.wait_event(done_reading[k])
            c_in.copy_(calib_h, non_blocking=True)
            w_in.copy_(W_h, non_blocking=True)
            x_in.copy_(X_h, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(h2d_stream)
        stream.wait_event(loaded)
        if done_writing[k] is not None:
            stream.wait_event(done_writing[k])
        step(bufs=sets[k])
        computed = torch.cuda.Event()
        computed.record(stream)
        done_reading[k] = computed
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(computed)
            y_hs[k].copy_(y_out, non_blocking=True)
            written = torch.cuda.Event()
            written.record(d2h_stream)
        done_writing[k] = written

    if e2e_steps:
        for i in range(2):
            e2e_step(i)
    barrier()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_stream.wait_stream(stream)
    d2h_stream.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(d2h_stream)
    stream.wait_stream(h2d_stream)
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps if e2e_steps else float("nan")
    if e2e_steps:
        # the last step's output arrived on the host intact
        if not torch.equal(y_hs[(e2e_steps - 1) % 2], y.cpu()):
            raise RuntimeError("end-to-end output differs from the device-resident step's output")
    te = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(te, op=dist.ReduceOp.MAX)
    e2e_ms = float(te.item())
    h2d = (calib.numel() + W.numel() + X.numel()) * 2 if e2e_steps else 0
    d2h = y.numel() * 2 if e2e_steps else 0

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    int8_peak = float(peaks["bf16_tflops"]) * INT8_PER_BF16
    work = stage_work(w, T, N, K, w.calib_rows)
    stages = {}
    for n in names:
        ms = stage_ms[n]
        wk = work[n]
        ent = {"ms": ms, "launches": LAUNCHES[n], "timed": "live" if n == names[dom_i] else "breakdown pass"}
        if wk["bound"] == "tensor":
            ent["tops"] = wk["ops"] / (ms * 1e-3) / 1e12
            ent["frac_of_int8_peak"] = ent["tops"] / int8_peak
        ent["gbs"] = wk["bytes"] / (ms * 1e-3) / 1e9
        ent["frac_of_hbm"] = ent["gbs"] / hbm
        stages[n] = ent
    dom = names[dom_i]
    kern, srcfile = KERNEL_OF[dom]
    if work[dom]["bound"] == "tensor":
        roof = {"bound": "tensor", "achieved": stages[dom]["tops"], "peak": int8_peak, "unit": "TOPS",
                "frac": stages[dom]["tops"] / int8_peak}
        peak_note = f"int8 peak = {src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16:g} (nominal int8/bf16 ratio)"
    else:
        roof = {"bound": "hbm", "achieved": stages[dom]["gbs"], "peak": hbm, "unit": "GB/s",
                "frac": stages[dom]["gbs"] / hbm}
        peak_note = f"HBM peak = {src} copy bandwidth"
    roof["traffic"] = recorded_traffic(dom, srcfile)
    roof["kernel"] = kern
    roof["stage"] = dom
    roof["peak_source"] = peak_note

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        import oracle as orc
        cores = cpu_cores()
        orc.set_threads(cores)
        secs, sample, _ = oracle_step_seconds(w, 1.0 / 16)
        cpu = {"value": w.linear_ops() / secs / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": sample}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": w.name, "T": T, "K": K, "N": N, "calib_rows": w.calib_rows, "alpha": w.alpha,
                   "norm": w.norm, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2: each step reads the 537 MB calibration set"},
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": {"value": world * w.linear_ops() / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": sum(LAUNCHES.values()) * args.steps,
        "clocks": {"sm_mhz": clk["sm_mhz"], "sm_max_mhz": clk["sm_max_mhz"], "reasons": clk["reasons"],
                   "samples": clk["samples"]},
        "stages": stages,
        "stages_note": (f"the dominant stage is timed in the timed steps with events around it only; the others come "
                        f"from a separate pass of {nb} steps with an event at every stage boundary (those events "
                        f"add ~20 us per step, so they stay out of the timed steps)"),
        "gemm_tops": stages["gemm"]["tops"],
        "gemm_frac_of_int8_peak": stages["gemm"]["frac_of_int8_peak"],
        # the GEMM runs inside a long step: its fraction of the sustained (power-capped) reference too
        "gemm_frac_of_int8_sustained": (stages["gemm"]["tops"] / (float(peaks["bf16_tflops_sustained"]) * INT8_PER_BF16)
                                        if "bf16_tflops_sustained" in peaks else None),
        "quant_kernel_gbs": stages["act_quant"]["gbs"],
        "online_ms_per_step": stage_ms["act_quant"] + stage_ms["gemm"],
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed CPU oracle sample")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end measurement")
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
