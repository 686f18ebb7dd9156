"""The layer-error harness ("SmoothQuant and W8A8...", "One layer, measured").

CPU: the reference output and the error metric against closed forms. GPU: the sweep on the single
linear workload reproduces the qualitative findings the page reports (smoothing lowers both INT8
errors on outlier data; a static per-tensor scale is worse than per-token scales without smoothing;
FP8 E4M3 barely needs smoothing, and smoothed INT8 beats it), and its quantised product agrees with
the bf16 output the layer returns.
"""
import numpy as np
import pytest
import torch

from post_quantization_calib_b200 import error_sweep


def test_reference_output_closed_form():
    # a constant row normalises to ones: RMSNorm(c) = c / |c| (eps -> 0), times gamma, times W
    x = torch.full((2, 8), 3.0, dtype=torch.bfloat16)
    x[1] = -0.5
    g = torch.linspace(0.5, 2.0, 8)
    w = torch.arange(24, dtype=torch.float32).reshape(3, 8) / 10
    ref = error_sweep.reference_output(x, w, g, eps=0.0)
    expect = torch.stack([g.double() @ w.double().t(), -(g.double() @ w.double().t())])
    assert torch.allclose(ref, expect, rtol=1e-15, atol=1e-15)
    # without gamma the input is x itself
    assert torch.equal(error_sweep.reference_output(x, w, None, 1e-6), x.double() @ w.double().t())


def test_relative_error_metric():
    a = torch.tensor([[3.0, 4.0]], dtype=torch.float64)
    assert error_sweep.relative_error(a, a) == 0.0
    assert abs(error_sweep.relative_error(a, torch.zeros(1, 2)) - 1.0) < 1e-15
    assert abs(error_sweep.relative_error(a, torch.tensor([[3.0, 3.0]])) - 0.2) < 1e-15   # |(0,1)| / 5


@pytest.mark.gpu
def test_sweep_single_linear_findings():
    rows = error_sweep.sweep("single_linear_t256_k1024_n1024", holdout=256, alphas=(0.5, 0.8))
    get = {(r["alpha"], r["scheme"]): r for r in rows}
    for scheme in ("per_token", "per_tensor"):
        base = get[(None, scheme)]["error"]
        assert get[(0.5, scheme)]["error"] < 0.7 * base, f"smoothing did not lower the {scheme} error"
        for r in rows:
            assert 0.0 < r["error"] < 0.5 and 0.0 < r["error_bf16"] < 0.5
            # the bf16 output differs from the exact dequantised product by bf16 rounding only
            assert abs(r["error_bf16"] - r["error"]) < 4e-3
    assert get[(None, "per_tensor")]["error"] > get[(None, "per_token")]["error"]
    s = error_sweep.summary(rows)
    assert s["per_tensor"]["reduction"] > 1.5 and s["per_token"]["reduction"] > 1.2
    # FP8: smoothing changes little, and smoothed INT8 per token beats the best FP8 point
    assert s["fp8_per_token"]["reduction"] < 1.3
    assert s["per_token"]["best"] < s["fp8_per_token"]["best"]


def _h16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


@pytest.mark.gpu
@pytest.mark.parametrize("workload,holdout", [("single_linear_t256_k1024_n1024", 256), ("qproj_t8192_k4096_n4096", 256)])
def test_sweep_matches_oracle_chain(orc, workload, holdout):
    """The harness's error figures recomputed from the CPU oracle on the same inputs: the oracle's
    calibration maxima, smoothing factors, weight and activation quantisers (per token and static
    per tensor) and INT8 GEMM, with the layer input and X W taken here in numpy binary64. The INT8
    accumulators are exact and every step is bit-exact against the oracle, so the two error figures
    (from the accumulators, and of the bf16 output) agree to rounding of the binary64 norms (1e-9
    relative). The FP8 point uses binary32 tensor-core accumulators: its figure agrees within the
    binary32 summation bound of the accumulators. The oracle is fed the library's smoothing factors
    (which match its own within the 1e-6 bar), as in the stage-by-stage parity tests, so that the bar
    on s cannot turn into code differences."""
    from post_quantization_calib_b200 import sq, synth
    alphas = (0.3, 0.5, 0.8)
    rows = error_sweep.sweep(workload, holdout=holdout, alphas=alphas)
    got = {(r["alpha"], r["scheme"]): r for r in rows}
    w = synth.workload(workload)
    d = synth.group_inputs(w, 0, "cuda")
    gamma = d["gamma"] if w.norm else None
    W, X = d["weight"], d["x"][:holdout]
    K = W.shape[1]
    g_h = None if gamma is None else gamma.cpu().numpy()
    chunks = list(synth.calibration_chunks(w, d["channels"], "cuda"))
    ch_h = [_h16(c) for c in chunks]
    W_h, X_h = _h16(W), _h16(X)
    amax_o = None
    for i, c in enumerate(ch_h):
        amax_o = orc.calibrate_absmax(c, norm_gamma=g_h, eps=w.eps, amax=amax_o, accumulate=i > 0)
    aw_o = orc.calibrate_absmax(W_h)
    amax_g = torch.empty(K, dtype=torch.float32, device="cuda")
    for i, c in enumerate(chunks):
        sq.sq_calibrate_absmax(c, norm_gamma=gamma, eps=w.eps, amax=amax_g, accumulate=i > 0)
    aw_g = sq.sq_calibrate_absmax(W)
    assert np.array_equal(amax_g.cpu().numpy(), amax_o) and np.array_equal(aw_g.cpu().numpy(), aw_o)
    # X W in binary64, X the layer's input
    x64 = _f64(X_h)
    if g_h is not None:
        x64 = x64 / np.sqrt((x64 * x64).mean(axis=1, keepdims=True) + w.eps) * g_h.astype(np.float64)
    ref = x64 @ _f64(W_h).T
    nref = np.linalg.norm(ref)
    table = orc.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)
    for a in (None,) + alphas:
        if a is None:
            s_h, f_h = None, (g_h.copy() if g_h is not None else np.ones(K, np.float32))
        else:
            s_o, f_o = orc.compute_scales(amax_o, aw_o, a, g_h)
            s_g, f_g = sq.sq_compute_scales(amax_g, aw_g, a, gamma=gamma)
            s_h, f_h = s_g.cpu().numpy(), f_g.cpu().numpy()
            assert np.all(np.abs(s_h.astype(np.float64) / s_o - 1) <= 1e-6)
            assert np.all(np.abs(f_h.astype(np.float64) / f_o - 1) <= 1e-6)
        wq, ws = orc.smooth_quantize_weight(W_h, s_h)
        for scheme in ("per_token", "per_tensor"):
            if scheme == "per_token":
                xq, xs = orc.rmsnorm_smooth_quant(X_h, f_h, eps=w.eps, apply_norm=w.norm)
            else:
                amax_y = None
                for i, c in enumerate(ch_h):
                    if w.norm:
                        amax_y = orc.calibrate_absmax(c, norm_gamma=f_h, eps=w.eps, amax=amax_y, accumulate=i > 0)
                    else:
                        amax_y = orc.calibrate_absmax(c, amax=amax_y, accumulate=i > 0)
                if not w.norm:
                    amax_y = (amax_y * np.abs(f_h)).astype(np.float32)
                xq, xs = orc.rmsnorm_smooth_quant_static(X_h, f_h, orc.static_scale(amax_y), eps=w.eps,
                                                         apply_norm=w.norm)
            y, acc = orc.w8a8_linear(xq, xs, wq, ws)
            qq = acc.astype(np.float64) * xs.astype(np.float64)[:, None] * ws.astype(np.float64)[None, :]
            e, eb = np.linalg.norm(ref - qq) / nref, np.linalg.norm(ref - _f64(y)) / nref
            r = got[(a, scheme)]
            assert abs(r["error"] / e - 1) <= 1e-9, (a, scheme, r["error"], e)
            assert abs(r["error_bf16"] / eb - 1) <= 1e-9, (a, scheme, r["error_bf16"], eb)
        wq8, ws8 = orc.smooth_quantize_weight_f8(W_h, s_h)
        xq8, xs8 = orc.rmsnorm_smooth_quant_f8(X_h, f_h, eps=w.eps, apply_norm=w.norm)
        exact = orc.gemm_f8(xq8, wq8)
        sc = xs8.astype(np.float64)[:, None] * ws8.astype(np.float64)[None, :]
        e8 = np.linalg.norm(ref - exact * sc) / nref
        mag = (np.abs(table[xq8]) @ np.abs(table[wq8]).T) * sc        # |products|, scaled
        bound = np.linalg.norm(K * 2.0 ** -24 * mag) / nref                # binary32 summation of the accumulators
        assert abs(got[(a, "fp8_per_token")]["error"] - e8) <= bound + 1e-12 * e8, (a, got[(a, "fp8_per_token")]["error"], e8, bound)
