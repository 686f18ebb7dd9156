"""Alpha sweep of the smoothed W8A8 layer's output error (the layer-error harness).

"SmoothQuant and W8A8: Quantizing Activations Too", "One layer, measured": the migration strength
alpha is swept from 0.1 to 1, plus a point without smoothing, with weights quantised per output
channel and activations either with one static scale per tensor (from the calibration maximum) or
one dynamic scale per token, in INT8 and in FP8 E4M3; the error is measured on the layer's output
for held-out tokens as
||X W - Q(X) Q(W)|| / ||X W|| (Frobenius norms).

Every quantisation step runs through the library (``sq``): calibration abs-maxima, smoothing factors
and fold, the smoothed INT8 weight, the activation quantiser (per token, or the static per-tensor
scale with its clipping quantiser) and the INT8 GEMM, whose exact INT32 accumulators give
Q(X) Q(W) = acc * x_scale[t] * w_scale[n] in binary64; the FP8 points use the E4M3 quantisers and the
FP8 GEMM (binary32 accumulators). The reference X W is the layer's input (the
RMSNorm output times gamma for a norm-fed layer, else x) times the weight, in binary64. The error of
the bf16 output the layer actually returns is reported beside it.

Run:  python -m post_quantization_calib_b200.error_sweep [--workload NAME] [--holdout 2048]
"""
from __future__ import annotations

import argparse
import json
from typing import Dict, List, Optional, Sequence

import torch

from . import synth

ALPHAS = tuple(round(0.1 * i, 1) for i in range(1, 11))


def reference_output(x: torch.Tensor, w: torch.Tensor, gamma: Optional[torch.Tensor], eps: float) -> torch.Tensor:
    """X W in binary64, X the layer's input: RMSNorm(x) * gamma when gamma is given, else x."""
    x64 = x.to(torch.float64)
    if gamma is not None:
        x64 = x64 * torch.rsqrt((x64 * x64).mean(dim=1, keepdim=True) + eps) * gamma.to(torch.float64)
    return x64 @ w.to(torch.float64).t()


def relative_error(ref: torch.Tensor, out: torch.Tensor) -> float:
    """||ref - out||_F / ||ref||_F in binary64."""
    d = ref - out.to(torch.float64)
    return float(torch.linalg.vector_norm(d) / torch.linalg.vector_norm(ref))


def sweep(workload: str = "qproj_t8192_k4096_n4096", holdout: int = 2048, alphas: Sequence[float] = ALPHAS,
          device: str = "cuda") -> List[Dict]:
    """One row per (smoothing point, activation scheme): alpha (None = unsmoothed), scheme
    ("per_token" | "per_tensor" INT8, "fp8_per_token" E4M3), error (from the accumulators: exact for
    INT8, binary32 for FP8) and error_bf16 (the bf16 output)."""
    from . import sq

    w = synth.workload(workload)
    d = synth.group_inputs(w, 0, device)
    gamma = d["gamma"] if w.norm else None
    W, X = d["weight"], d["x"][:holdout]
    T, K = X.shape
    N = W.shape[0]
    ref = reference_output(X, W, gamma, w.eps)

    # calibration abs-maxima (alpha independent), streamed over the calibration chunks
    amax = torch.empty(K, dtype=torch.float32, device=device)
    chunks = list(synth.calibration_chunks(w, d["channels"], device))
    for i, c in enumerate(chunks):
        sq.sq_calibrate_absmax(c, norm_gamma=gamma, eps=w.eps, amax=amax, accumulate=i > 0)
    aw = sq.sq_calibrate_absmax(W)

    acc = torch.empty(T, N, dtype=torch.int32, device=device)
    accf = torch.empty(T, N, dtype=torch.float32, device=device)
    rows: List[Dict] = []
    points: List[Optional[float]] = [None] + [float(a) for a in alphas]
    for a in points:
        if a is None:       # unsmoothed: s = 1, the fold is gamma itself (or 1)
            s = None
            fold = gamma.clone() if gamma is not None else torch.ones(K, dtype=torch.float32, device=device)
        else:
            s, fold = sq.sq_compute_scales(amax, aw, a, gamma=gamma)
        wq, ws = sq.sq_smooth_quantize_weight(W, s)
        wq8, ws8 = sq.sq_smooth_quantize_weight_fp8(W, s)
        for scheme in ("per_token", "per_tensor", "fp8_per_token"):
            if scheme == "fp8_per_token":
                xq8, xs8 = sq.sq_rmsnorm_smooth_quant_fp8(X, fold, eps=w.eps, apply_norm=w.norm)
                y = sq.sq_w8a8_linear_fp8(xq8, xs8, wq8, ws8, acc_out=accf)
                qq = accf.to(torch.float64) * xs8.to(torch.float64)[:, None] * ws8.to(torch.float64)[None, :]
                rows.append({"workload": workload, "alpha": a, "scheme": scheme, "tokens": T,
                             "error": relative_error(ref, qq), "error_bf16": relative_error(ref, y)})
                continue
            if scheme == "per_token":
                xq, xs = sq.sq_rmsnorm_smooth_quant(X, fold, eps=w.eps, apply_norm=w.norm)
            else:
                amax_y = torch.empty(K, dtype=torch.float32, device=device)
                if w.norm:
                    for i, c in enumerate(chunks):
                        sq.sq_calibrate_absmax(c, norm_gamma=fold, eps=w.eps, amax=amax_y, accumulate=i > 0)
                    s2 = sq.sq_static_scale(amax_y)
                else:
                    for i, c in enumerate(chunks):
                        sq.sq_calibrate_absmax(c, amax=amax_y, accumulate=i > 0)
                    s2 = sq.sq_static_scale(amax_y, factor=fold)
                xq, xs = sq.sq_rmsnorm_smooth_quant_static(X, fold, s2, eps=w.eps, apply_norm=w.norm)
            y = sq.sq_w8a8_linear(xq, xs, wq, ws, acc_out=acc)
            qq = acc.to(torch.float64) * xs.to(torch.float64)[:, None] * ws.to(torch.float64)[None, :]
            rows.append({"workload": workload, "alpha": a, "scheme": scheme, "tokens": T,
                         "error": relative_error(ref, qq), "error_bf16": relative_error(ref, y)})
    return rows


def summary(rows: List[Dict]) -> Dict:
    """Unsmoothed vs best smoothed error per scheme, and the alpha that gives it."""
    out = {}
    for scheme in ("per_token", "per_tensor", "fp8_per_token"):
        r = [x for x in rows if x["scheme"] == scheme]
        base = next(x for x in r if x["alpha"] is None)
        best = min((x for x in r if x["alpha"] is not None), key=lambda x: x["error"])
        out[scheme] = {"unsmoothed": base["error"], "best": best["error"], "best_alpha": best["alpha"],
                       "reduction": base["error"] / best["error"]}
    return out


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", default="qproj_t8192_k4096_n4096")
    ap.add_argument("--holdout", type=int, default=2048)
    args = ap.parse_args(argv)
    rows = sweep(args.workload, args.holdout)
    for r in rows:
        print(json.dumps(r))
    print(json.dumps({"summary": summary(rows)}))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
