"""Per-workload report: every stage's GPU time and rate beside its parity against the CPU oracle and
the oracle's own time on the same inputs (test infrastructure: it calls the oracle).

    python tests/parity_report.py [--workload NAME ...] [--reps 20] [--gemm-sample 24]

One JSON line per workload, smoothing group and stage (the stages of the benchmark's step):
  calib_absmax_pair  S1 + S2  abs-maxima of the calibration set (RMSNorm output when norm-fed) and the
                              weight, one launch; parity: mismatching channels (bit-exact bar)
  scales             S3       s and the fold; parity: largest relative error (bar 1e-6)
  weight_quant       S4       INT8 weight codes and scales; parity: mismatching codes / scales
  act_quant          S5       per-token INT8 codes and scales; parity: mismatching codes / scales
  gemm               S6 + S7  INT32 accumulators and bf16 outputs on sampled full rows and full columns;
                              parity: mismatching accumulators, outputs differing from the oracle's
                              epilogue, largest relative error against the exact dequantised value
Each stage is fed the GPU's own earlier outputs on both sides (as in the parity tests). GPU times are
medians of CUDA-event single calls with the L2 cleared before each (``perf.Timer``); oracle times are
measured on the stage's full input, except the GEMM, which the oracle runs only on the sampled rows
and columns: its full time is extrapolated from them (labelled). The oracle's GEMM runs on all host
cores (OpenMP); its other stages run on one thread, so the activation quantiser's time is a one-thread
figure.
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from post_quantization_calib_b200 import perf, synth  # noqa: E402


def h16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def hn(t):
    return t.detach().contiguous().cpu().numpy()


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def timed(fn):
    t0 = time.perf_counter()
    out = fn()
    return out, time.perf_counter() - t0


def sample_indices(n, k, seed):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=min(k, n), replace=False).tolist()) | {0, n - 1}
    return np.array(sorted(pick), np.int64)


def report_group(w, g, timer, peaks, gemm_sample, cores):
    from post_quantization_calib_b200 import sq
    import oracle as orc
    dev = "cuda"
    out = []
    d = synth.group_inputs(w, g, dev)
    gamma, W, X, bias = d["gamma"], d["weight"], d["x"], d["bias"]
    N, K = W.shape
    T = X.shape[0]
    g_h = None if gamma is None else hn(gamma)
    calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], dev, group=g)))
    R = calib.shape[0]
    base = {"workload": w.name, "group": g}

    def line(stage, us, nbytes, ops=None, **kw):
        r = perf.line(peaks, w.name, g, stage, us, nbytes, ops)
        r.update(kw)
        out.append(r)
        print(json.dumps(r), flush=True)

    # S1 + S2
    amax = torch.empty(K, dtype=torch.float32, device=dev)
    aw = torch.empty(K, dtype=torch.float32, device=dev)
    pair = lambda: sq.sq_calibrate_absmax_pair(calib, W, norm_gamma=gamma, eps=w.eps, amax=amax, amax_w=aw)
    us = timer.single(pair)
    c_h, w_h = h16(calib), h16(W)
    amax_o, t1 = timed(lambda: orc.calibrate_absmax(c_h, norm_gamma=g_h, eps=w.eps))
    aw_o, t2 = timed(lambda: orc.calibrate_absmax(w_h))
    mism = int((hn(amax) != amax_o).sum() + (hn(aw) != aw_o).sum())
    line("calib_absmax_pair", us, 2 * R * K + 2 * N * K + 12 * K, rows=R, N=N, K=K, mismatches=mism,
         checked=f"all {2 * K} channels", oracle_s=t1 + t2, oracle_threads=1)
    del c_h
    # S3
    s = torch.empty(K, dtype=torch.float32, device=dev)
    fold = torch.empty(K, dtype=torch.float32, device=dev)
    us = timer.single(lambda: sq.sq_compute_scales(amax, aw, w.alpha, gamma=gamma, s=s, fold=fold))
    (s_o, f_o), t3 = timed(lambda: orc.compute_scales(hn(amax), hn(aw), w.alpha, g_h))
    rel = max(float(np.max(np.abs(hn(s).astype(np.float64) / s_o - 1))),
              float(np.max(np.abs(hn(fold).astype(np.float64) / f_o - 1))))
    line("scales", us, 20 * K, K=K, max_rel_err=rel, bar=1e-6, checked=f"all {K} channels", oracle_s=t3, oracle_threads=1)
    # S4 (oracle fed the GPU's s)
    wq = torch.empty(N, K, dtype=torch.int8, device=dev)
    ws = torch.empty(N, dtype=torch.float32, device=dev)
    us = timer.single(lambda: sq.sq_smooth_quantize_weight(W, s, wq=wq, w_scale=ws))
    (wq_o, ws_o), t4 = timed(lambda: orc.smooth_quantize_weight(w_h, hn(s)))
    line("weight_quant", us, 3 * N * K + 4 * K + 4 * N, N=N, K=K, mismatches=int((hn(wq) != wq_o).sum()),
         scale_mismatches=int((hn(ws) != ws_o).sum()), checked=f"all {N * K} codes", oracle_s=t4, oracle_threads=1)
    # S5 (oracle fed the GPU's fold)
    xq = torch.empty(T, K, dtype=torch.int8, device=dev)
    xs = torch.empty(T, dtype=torch.float32, device=dev)
    us = timer.single(lambda: sq.sq_rmsnorm_smooth_quant(X, fold, eps=w.eps, apply_norm=w.norm, xq=xq, x_scale=xs))
    x_h = h16(X)
    (xq_o, xs_o), t5 = timed(lambda: orc.rmsnorm_smooth_quant(x_h, hn(fold), eps=w.eps, apply_norm=w.norm))
    line("act_quant", us, 3 * T * K + 4 * K + 4 * T, T=T, K=K, mismatches=int((hn(xq) != xq_o).sum()),
         scale_mismatches=int((hn(xs) != xs_o).sum()), checked=f"all {T * K} codes", oracle_s=t5, oracle_threads=1)
    # S6 + S7 on sampled full rows and full columns
    y = torch.empty(T, N, dtype=torch.bfloat16, device=dev)
    us = timer.single(lambda: sq.sq_w8a8_linear(xq, xs, wq, ws, bias=bias, y=y))
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    sq.sq_w8a8_linear(xq, xs, wq, ws, bias=bias, y=y, acc_out=acc)
    rows, cols = sample_indices(T, gemm_sample, 7 + g), sample_indices(N, gemm_sample, 11 + g)
    b_h = None if bias is None else h16(bias)
    xq_h, wq_h, xs_h, ws_h = hn(xq), hn(wq), hn(xs), hn(ws)
    macc = my = 0
    rel = 0.0
    t6 = 0.0
    for sel_r, sel_c in ((rows, None), (None, cols)):
        (y_o, acc_o), dt = timed(lambda: orc.w8a8_linear(xq_h, xs_h, wq_h, ws_h, b_h, sel_r, sel_c))
        t6 += dt
        a_g, y_g = acc, y
        if sel_r is not None:
            ri = torch.as_tensor(sel_r, device=dev)
            a_g, y_g = a_g.index_select(0, ri), y_g.index_select(0, ri)
        if sel_c is not None:
            ci = torch.as_tensor(sel_c, device=dev)
            a_g, y_g = a_g.index_select(1, ci), y_g.index_select(1, ci)
        a_g, y_g = hn(a_g), h16(y_g)
        macc += int((a_g != acc_o).sum())
        my += int((y_g != y_o).sum())
        rs = slice(None) if sel_r is None else sel_r
        cs = slice(None) if sel_c is None else sel_c
        exact = acc_o.astype(np.float64) * xs_h[rs][:, None].astype(np.float64) * ws_h[cs][None, :]
        ref = exact + (f64(b_h[cs])[None, :] if b_h is not None else 0.0)
        nz = np.abs(ref) > 0
        if nz.any():
            rel = max(rel, float(np.max(np.abs(f64(y_g)[nz] - ref[nz]) / np.abs(ref[nz]))))
    units = len(rows) * N + T * len(cols)
    line("gemm", us, T * K + N * K + 2 * T * N + 4 * T + 4 * N, 2 * T * N * K, T=T, N=N, K=K,
         acc_mismatches=macc, y_mismatches=my, max_rel_err=rel, bar=1e-2,
         checked=f"{len(rows)} full rows and {len(cols)} full columns", oracle_s=t6 * (T * N) / units,
         oracle_extrapolated=True, oracle_threads=cores)
    del calib
    torch.cuda.empty_cache()
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", action="append", help="workload name (repeatable; default: all five)")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--gemm-sample", type=int, default=24)
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        print("parity_report: needs a CUDA device", file=sys.stderr)
        return 2
    import oracle as orc
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    orc.set_threads(cores)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = perf.load_peaks()
    timer = perf.Timer(dev, args.reps)
    bad = 0
    for n in args.workload or [w.name for w in synth.WORKLOADS]:
        w = synth.workload(n)
        for g in range(w.groups):
            for r in report_group(w, g, timer, peaks, args.gemm_sample, cores):
                bad += r.get("mismatches", 0) + r.get("scale_mismatches", 0) + r.get("acc_mismatches", 0) + \
                    r.get("y_mismatches", 0) + (1 if r.get("max_rel_err", 0) > r.get("bar", 1) else 0)
    return 1 if bad else 0


if __name__ == "__main__":
    sys.exit(main())
