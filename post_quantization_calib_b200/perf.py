"""Per-workload timing of every stage of the smoothed W8A8 path: one JSON line per workload, group and stage.

    python -m post_quantization_calib_b200.perf [--workload NAME ...] [--stage NAME ...] [--tokens T ...]
                                                [--reps 20]

Each stage runs through the C ABI on the workload's seeded synthetic inputs (``synth``), resident in HBM:
  calib_absmax_pair  S1 + S2: column abs-max of the calibration set (of its RMSNorm output when norm-fed)
                     and of the group's weight, one launch
  scales             S3: smoothing factors and the folded norm weight
  weight_quant       S4: diag(s) W quantised to INT8 per output channel
  act_quant          S5: fused RMSNorm(gamma / s) + per-token INT8 of the workload's T tokens
  gemm               S6 + S7: INT8 GEMM with the dequant epilogue to bf16
The variant paths are timed only when named with --stage: act_quant_static (static per-tensor scale),
act_quant_fp8 and weight_quant_fp8 (E4M3 codes), gemm_fp8 (kind::f8f6f4 GEMM), act_quant_layernorm
(LayerNorm with gamma / s and beta / s folded), calib_absmax_layernorm (abs-max of the calibration set's
LayerNorm output) and fold_prev_linear (1/s folded into a previous [K, N] linear layer and its bias).
Decode workloads add act_quant and gemm at each decode token count, once as a single call and once per
call in a chain of 8 back-to-back calls captured in a CUDA graph (the way a decoder runs one layer after
another, without the host's per-call cost; the 8 GEMMs read 8 distinct copies of the weight, which
together exceed the L2). The GEMM chain is also timed issued call by call on the stream ("chain_form":
"stream"), where each call's dependent launch overlaps the previous call's end, and whole decode layers
(the activation quantiser, then the GEMM, 8 layers in one graph: stage "layer", per layer). The HBM-bound stages
(calib_absmax_pair, weight_quant, act_quant) are likewise timed per call in a CUDA graph of 8 calls on 8
copies of their inputs ("chain": 8), unless --no-chain is given.

Times are medians of CUDA-event intervals on the launching stream, with the L2 flushed (a 256 MB read)
before every repetition. Rates are algorithmic bytes (or 2 x multiply-adds) over that
time, also given as fractions of the HBM copy bandwidth and of the dense INT8 reference (2 x the bf16
GEMM burst) measured on the machine (``MEASURED_PEAKS.json`` at the repository root; else a fallback
pair, marked as such).
"""
from __future__ import annotations

import argparse
import json
import os
import sys
from typing import Callable, Dict, List, Optional

import torch

from . import sq, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
INT8_PER_BF16 = 2.0          # nominal dense INT8 / bf16 tensor throughput of the B200


def load_peaks() -> Dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


class Timer:
    """CUDA-event medians on the current stream, L2 flushed before each repetition by reading a 256 MB
    buffer (a read leaves clean lines, so no write-back of the flush lands inside the timed call).

    With `hold` (the default) a spin kernel of about 100 us follows the flush, so that the host has
    queued the timed call before the first event fires: the interval is then the call's device time
    (its launch on the device included), not the host's marshalling and launch cost."""

    HOLD_CYCLES = 200_000

    def __init__(self, device, reps: int, hold: bool = True):
        self.reps = reps
        self.hold = hold
        self.flush = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)

    def clear_l2(self) -> None:
        torch.sum(self.flush, dim=0, out=self.sink)
        if self.hold:
            torch.cuda._sleep(self.HOLD_CYCLES)

    def single(self, fn: Callable[[], None]) -> float:
        fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(self.reps)]
        for a, b in ev:
            self.clear_l2()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        t = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
        return t[len(t) // 2]

    def stream_chained(self, fns: List[Callable[[], None]]) -> float:
        """Microseconds per call of the calls `fns` issued back to back on the stream (each call may
        start while the previous one finishes), median over the repetitions. Only meaningful where a
        call takes longer on the device than on the host."""
        for fn in fns:
            fn()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(self.reps)]
        for a, b in ev:
            self.clear_l2()
            a.record()
            for fn in fns:
                fn()
            b.record()
        torch.cuda.synchronize()
        t = sorted(a.elapsed_time(b) * 1e3 / len(fns) for a, b in ev)
        return t[len(t) // 2]

    def chained(self, fns: List[Callable[[], None]]) -> float:
        """Microseconds per call of the calls `fns`, back to back, captured in one CUDA graph (so that
        the host's per-call cost does not enter), median over the repetitions."""
        calls = len(fns)
        fns[0]()                               # first call: the library's per-device set-up
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(graph, stream=side):
            for fn in fns:
                fn()
        graph.replay()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(self.reps)]
        for a, b in ev:
            self.clear_l2()
            a.record()
            graph.replay()
            b.record()
        torch.cuda.synchronize()
        t = sorted(a.elapsed_time(b) * 1e3 / calls for a, b in ev)
        return t[len(t) // 2]


def line(peaks: Dict, workload: str, group: int, stage: str, us: float, nbytes: int,
         ops: Optional[int] = None, **extra) -> Dict:
    out = {"workload": workload, "group": group, "stage": stage, **extra, "us": round(us, 2),
           "gbs": round(nbytes / us / 1e3, 1), "frac_hbm": round(nbytes / us / 1e3 / peaks["hbm_gbs"], 3)}
    if ops is not None:
        int8 = peaks["bf16_tflops"] * INT8_PER_BF16
        out["tops"] = round(ops / us / 1e6, 1)
        out["frac_int8"] = round(ops / us / 1e6 / int8, 3)
    out["peaks"] = peaks["source"]
    return out


STAGES = ("calib_absmax_pair", "scales", "weight_quant", "act_quant", "gemm")
# Variant paths, timed only when asked for (--stage): the static per-tensor activation quantiser (its
# scale from the calibration abs-max of the quantiser's own y), the FP8 E4M3 per-token quantiser, the
# LayerNorm-fed quantiser (gamma and beta folded; the tokens' own LayerNorm stands in for the RMSNorm),
# the FP8 weight quantiser and the FP8 GEMM; the LayerNorm calibration abs-max and the fold of 1/s into
# a previous linear layer (a [K, N] weight and bias: the layer whose output feeds this one), both timed
# once per group.
VARIANTS = ("act_quant_static", "act_quant_fp8", "act_quant_layernorm", "weight_quant_fp8", "gemm_fp8",
            "calib_absmax_layernorm", "fold_prev_linear")


CHAIN = 8   # calls per timed chain (each on its own copy of the inputs, together beyond the L2)


def run_workload(w: synth.Workload, timer: Timer, peaks: Dict, device, stages=STAGES,
                 tokens: Optional[List[int]] = None, chain: bool = True) -> List[Dict]:
    """The workload's stages (those in `stages`; the others still run once, untimed, where a later
    stage needs their output), at the workload's token count and its decode token counts (or at
    `tokens`). With `chain`, the HBM-bound stages at the workload's own token count are also timed per
    call in a CUDA graph of CHAIN calls on distinct copies of their inputs ("chain": CHAIN): the way
    they run inside a model, without the fixed cost of one event-timed launch."""
    rows: List[Dict] = []
    K = w.K
    for g in range(w.groups):
        N = w.group_N(g)
        d = synth.group_inputs(w, g, device)
        gamma, W, X, bias = d["gamma"], d["weight"], d["x"], d["bias"]
        calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], device, group=g)))
        R = calib.shape[0]
        amax = torch.empty(K, dtype=torch.float32, device=device)
        aw = torch.empty(K, dtype=torch.float32, device=device)
        pair = lambda: sq.sq_calibrate_absmax_pair(calib, W, norm_gamma=gamma, eps=w.eps, amax=amax, amax_w=aw)
        if "calib_absmax_pair" in stages:
            pbytes = 2 * R * K + 2 * N * K + 12 * K
            rows.append(line(peaks, w.name, g, "calib_absmax_pair", timer.single(pair), pbytes, rows=R, N=N, K=K))
            if chain:
                copies = [(calib, W)] + [(calib.clone(), W.clone()) for _ in range(CHAIN - 1)]
                fns = [lambda c=c, m=m: sq.sq_calibrate_absmax_pair(c, m, norm_gamma=gamma, eps=w.eps, amax=amax, amax_w=aw)
                       for c, m in copies]
                rows.append(line(peaks, w.name, g, "calib_absmax_pair", timer.chained(fns), pbytes, rows=R, N=N, K=K,
                                 chain=CHAIN))
                del copies, fns
                torch.cuda.empty_cache()
        pair()
        s = torch.empty(K, dtype=torch.float32, device=device)
        fold = torch.empty(K, dtype=torch.float32, device=device)
        scales = lambda: sq.sq_compute_scales(amax, aw, w.alpha, gamma=gamma, s=s, fold=fold)
        if "scales" in stages:
            rows.append(line(peaks, w.name, g, "scales", timer.single(scales), 20 * K, K=K))
        else:
            scales()
        wq = torch.empty(N, K, dtype=torch.int8, device=device)
        ws = torch.empty(N, dtype=torch.float32, device=device)
        wquant = lambda: sq.sq_smooth_quantize_weight(W, s, wq=wq, w_scale=ws)
        if "weight_quant" in stages:
            wbytes = 3 * N * K + 4 * K + 4 * N
            rows.append(line(peaks, w.name, g, "weight_quant", timer.single(wquant), wbytes, N=N, K=K))
            if chain:
                copies = [W] + [W.clone() for _ in range(CHAIN - 1)]
                fns = [lambda m=m: sq.sq_smooth_quantize_weight(m, s, wq=wq, w_scale=ws) for m in copies]
                rows.append(line(peaks, w.name, g, "weight_quant", timer.chained(fns), wbytes, N=N, K=K, chain=CHAIN))
                del copies, fns
                torch.cuda.empty_cache()
        wquant()
        token_counts = tokens if tokens else [w.T] + [t for t in w.decode_T if t != w.T]
        for T in token_counts:
            x = X[:T] if T <= X.shape[0] else synth.outlier_tokens(T, K, d["channels"], synth.seed_for(w.index, "x", g), device)
            xq = torch.empty(T, K, dtype=torch.int8, device=device)
            xs = torch.empty(T, dtype=torch.float32, device=device)
            y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
            quant = lambda: sq.sq_rmsnorm_smooth_quant(x, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs)
            gemm = lambda: sq.sq_w8a8_linear(xq, xs, wq, ws, bias=bias, y=y)
            qbytes = 3 * T * K + 4 * K + 4 * T
            gbytes = T * K + N * K + 2 * T * N + 4 * T + 4 * N + (2 * N if bias is not None else 0)
            ops = 2 * T * N * K
            if "act_quant" in stages:
                rows.append(line(peaks, w.name, g, "act_quant", timer.single(quant), qbytes, T=T, K=K))
                if chain and T == w.T and T not in w.decode_T:
                    copies = [x] + [x.clone() for _ in range(CHAIN - 1)]
                    fns = [lambda c=c: sq.sq_rmsnorm_smooth_quant(c, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs)
                           for c in copies]
                    rows.append(line(peaks, w.name, g, "act_quant", timer.chained(fns), qbytes, T=T, K=K, chain=CHAIN))
                    del copies, fns
            quant()
            if "gemm" in stages:
                rows.append(line(peaks, w.name, g, "gemm", timer.single(gemm), gbytes, ops, T=T, N=N, K=K))
            if any(v in stages for v in VARIANTS):
                rows.extend(run_variants(w, g, peaks, timer, stages, x, fold, W, s, calib, bias, gamma, T, N, K, device))
            if T in w.decode_T and "gemm" in stages and "act_quant" in stages:
                # a decoder's consecutive layers: each GEMM streams its own weight (8 together exceed
                # the L2); the activations are small and stay in L2 either way
                wqs = [wq] + [wq.clone() for _ in range(7)]
                gemms = [lambda m=m: sq.sq_w8a8_linear(xq, xs, m, ws, bias=bias, y=y) for m in wqs]
                rows.append(line(peaks, w.name, g, "act_quant", timer.chained([quant] * 8), qbytes, T=T, K=K, chain=8))
                rows.append(line(peaks, w.name, g, "gemm", timer.chained(gemms), gbytes, ops, T=T, N=N, K=K, chain=8))
                rows.append(line(peaks, w.name, g, "gemm", timer.stream_chained(gemms), gbytes, ops, T=T, N=N, K=K,
                                 chain=8, chain_form="stream"))
                # whole decode layers: each layer quantises its own tokens, then multiplies by its own weight
                xs8 = [x] + [x.clone() for _ in range(7)]
                quants = [lambda c=c: sq.sq_rmsnorm_smooth_quant(c, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs)
                          for c in xs8]
                layer = [f for pair in zip(quants, gemms) for f in pair]
                rows.append(line(peaks, w.name, g, "layer", 2 * timer.chained(layer), qbytes + gbytes, ops, T=T, N=N, K=K,
                                 chain=8, chain_form="layer"))
                del wqs, gemms, xs8, quants, layer
        del calib
        torch.cuda.empty_cache()
    st = sq.sq_device_status()
    if st != 0:
        raise RuntimeError(f"device status {sq.sq_status_string(st)} after workload {w.name}")
    return rows


def run_variants(w, g, peaks, timer, stages, x, fold, W, s, calib, bias, gamma, T, N, K, device) -> List[Dict]:
    """The variant paths at the workload's shapes (the stages named in VARIANTS that `stages` asks for)."""
    rows: List[Dict] = []
    qbytes = 3 * T * K + 4 * K + 4 * T
    xq = torch.empty(T, K, dtype=torch.int8, device=device)
    xs = torch.empty(T, dtype=torch.float32, device=device)
    if "act_quant_static" in stages:
        amax_y = torch.empty(K, dtype=torch.float32, device=device)
        if w.norm:
            sq.sq_calibrate_absmax(calib, norm_gamma=fold, eps=w.eps, amax=amax_y)
            s2 = sq.sq_static_scale(amax_y)
        else:
            sq.sq_calibrate_absmax(calib, amax=amax_y)
            s2 = sq.sq_static_scale(amax_y, factor=fold)
        f = lambda: sq.sq_rmsnorm_smooth_quant_static(x, fold, s2, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs)
        rows.append(line(peaks, w.name, g, "act_quant_static", timer.single(f), qbytes, T=T, K=K))
    if "act_quant_fp8" in stages or "gemm_fp8" in stages:
        xq8 = torch.empty(T, K, dtype=torch.uint8, device=device)
        xs8 = torch.empty(T, dtype=torch.float32, device=device)
        f = lambda: sq.sq_rmsnorm_smooth_quant_fp8(x, fold, eps=w.eps, apply_norm=w.norm, xq=xq8, x_scale=xs8)
        us = timer.single(f)
        if "act_quant_fp8" in stages:
            rows.append(line(peaks, w.name, g, "act_quant_fp8", us, qbytes, T=T, K=K))
    if "act_quant_layernorm" in stages:
        beta = 0.05 * torch.randn(K, generator=torch.Generator(device=device).manual_seed(7), device=device)
        g_ln = gamma if gamma is not None else torch.ones(K, dtype=torch.float32, device=device)
        f_ln = torch.empty(K, dtype=torch.float32, device=device)
        s_ln = torch.empty(K, dtype=torch.float32, device=device)
        amax_ln = sq.sq_calibrate_absmax_layernorm(calib, g_ln, beta)
        sq.sq_compute_scales(amax_ln, sq.sq_calibrate_absmax(W), w.alpha, gamma=g_ln, s=s_ln, fold=f_ln)
        bf = sq.sq_fold_layernorm_bias(beta, s_ln)
        f = lambda: sq.sq_layernorm_smooth_quant(x, f_ln, bf, xq=xq, x_scale=xs)
        rows.append(line(peaks, w.name, g, "act_quant_layernorm", timer.single(f), qbytes + 4 * K, T=T, K=K))
    if "weight_quant_fp8" in stages or "gemm_fp8" in stages:
        wq8 = torch.empty(N, K, dtype=torch.uint8, device=device)
        ws8 = torch.empty(N, dtype=torch.float32, device=device)
        f = lambda: sq.sq_smooth_quantize_weight_fp8(W, s, wq=wq8, w_scale=ws8)
        us = timer.single(f)
        if "weight_quant_fp8" in stages:
            rows.append(line(peaks, w.name, g, "weight_quant_fp8", us, 3 * N * K + 4 * K + 4 * N, N=N, K=K))
    if "gemm_fp8" in stages:
        y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
        f = lambda: sq.sq_w8a8_linear_fp8(xq8, xs8, wq8, ws8, bias=bias, y=y)
        gbytes = T * K + N * K + 2 * T * N + 4 * T + 4 * N + (2 * N if bias is not None else 0)
        rows.append(line(peaks, w.name, g, "gemm_fp8", timer.single(f), gbytes, 2 * T * N * K, T=T, N=N, K=K))
    if T == w.T and "calib_absmax_layernorm" in stages:
        g_ln = gamma if gamma is not None else torch.ones(K, dtype=torch.float32, device=device)
        beta = torch.zeros(K, dtype=torch.float32, device=device)
        amax_ln = torch.empty(K, dtype=torch.float32, device=device)
        f = lambda: sq.sq_calibrate_absmax_layernorm(calib, g_ln, beta, amax=amax_ln)
        R = calib.shape[0]
        rows.append(line(peaks, w.name, g, "calib_absmax_layernorm", timer.single(f), 2 * R * K + 12 * K,
                         rows=R, K=K))
    if T == w.T and "fold_prev_linear" in stages:
        gen = torch.Generator(device=device).manual_seed(11)
        wp = (0.02 * torch.randn(K, N, generator=gen, device=device)).to(torch.bfloat16)
        bp = (0.01 * torch.randn(K, generator=gen, device=device)).to(torch.bfloat16)
        wp_out = torch.empty_like(wp)
        bp_out = torch.empty_like(bp)
        f = lambda: sq.sq_fold_into_prev_linear(wp, fold, bp, w_out=wp_out, b_out=bp_out)
        rows.append(line(peaks, w.name, g, "fold_prev_linear", timer.single(f), 4 * K * N + 8 * K,
                         rows=K, cols=N))
        del wp, wp_out
    return rows


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", action="append", help="workload name (repeatable; default: all five)")
    ap.add_argument("--stage", action="append", choices=STAGES + VARIANTS,
                    help="stage to time (repeatable; default: the five stages of the path; the variants only when named)")
    ap.add_argument("--tokens", action="append", type=int, help="token count (repeatable; default: the workload's)")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--no-chain", action="store_true", help="single calls only (no chains of calls in a CUDA graph)")
    ap.add_argument("--no-hold", action="store_true",
                    help="no spin kernel between the flush and the timed call (the host's launch cost may then enter)")
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        print("perf: needs a CUDA device", file=sys.stderr)
        return 2
    device = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    timer = Timer(device, args.reps, hold=not args.no_hold)
    names = args.workload or [w.name for w in synth.WORKLOADS]
    for n in names:
        for r in run_workload(synth.workload(n), timer, peaks, device, stages=tuple(args.stage or STAGES),
                              tokens=args.tokens, chain=not args.no_chain):
            r["host_ahead"] = timer.hold
            print(json.dumps(r), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
