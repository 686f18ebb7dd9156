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
