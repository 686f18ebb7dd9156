"""The per-workload timing tool: one JSON line per stage with positive times and rates (GPU), and a clean
exit without a device (CPU)."""
import io
import json
from contextlib import redirect_stdout

import pytest
import torch


def test_perf_needs_a_device():
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    from post_quantization_calib_b200 import perf
    assert perf.main(["--workload", "single_linear_t256_k1024_n1024", "--reps", "2"]) == 2
    assert perf.main(["--stage", "gemm", "--tokens", "1", "--tokens", "64"]) == 2
    with pytest.raises(SystemExit):
        perf.main(["--stage", "not_a_stage"])


@pytest.mark.gpu
def test_perf_lines_for_the_smallest_and_the_decode_workload():
    from post_quantization_calib_b200 import build
    build.build()
    from post_quantization_calib_b200 import perf
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = perf.main(["--workload", "single_linear_t256_k1024_n1024", "--workload", "decode_k4096_n14336",
                        "--reps", "3"])
    assert rc == 0
    rows = [json.loads(l) for l in buf.getvalue().splitlines() if l.strip()]
    stages = {(r["workload"], r["stage"], r.get("T"), r.get("chain")) for r in rows}
    forms = {(r["stage"], r.get("T"), r.get("chain_form")) for r in rows if r.get("chain")}
    for st in ("calib_absmax_pair", "scales", "weight_quant"):
        assert ("single_linear_t256_k1024_n1024", st, None, None) in stages
    assert ("single_linear_t256_k1024_n1024", "gemm", 256, None) in stages
    for T in (1, 8, 32, 64):
        assert ("decode_k4096_n14336", "gemm", T, None) in stages
        assert ("decode_k4096_n14336", "gemm", T, 8) in stages
        assert ("decode_k4096_n14336", "act_quant", T, 8) in stages
        assert ("gemm", T, "stream") in forms and ("gemm", T, None) in forms
        assert ("layer", T, "layer") in forms
    # the HBM-bound stages of the small workload also per call in a chain of 8
    for st in ("calib_absmax_pair", "weight_quant", "act_quant"):
        assert any(r["workload"] == "single_linear_t256_k1024_n1024" and r["stage"] == st and r.get("chain") == 8
                   for r in rows)
    for r in rows:
        assert r["us"] > 0 and r["gbs"] > 0 and r["peaks"] in ("measured", "fallback")
        if r["stage"] == "gemm":
            assert r["tops"] > 0


@pytest.mark.gpu
def test_parity_report_lines_for_the_single_linear():
    """The per-workload report: every stage of the single linear layer with its GPU rate, its parity
    against the oracle (all bit-exact, the scale and bf16 bars met) and the oracle's time."""
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
    import parity_report
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = parity_report.main(["--workload", "single_linear_t256_k1024_n1024", "--reps", "3", "--gemm-sample", "8"])
    assert rc == 0
    rows = {r["stage"]: r for r in (json.loads(l) for l in buf.getvalue().splitlines() if l.strip())}
    assert set(rows) == {"calib_absmax_pair", "scales", "weight_quant", "act_quant", "gemm"}
    for st in ("calib_absmax_pair", "weight_quant", "act_quant"):
        assert rows[st]["mismatches"] == 0 and rows[st]["oracle_s"] > 0 and rows[st]["us"] > 0
    assert rows["scales"]["max_rel_err"] <= 1e-6
    g = rows["gemm"]
    assert g["acc_mismatches"] == 0 and g["y_mismatches"] == 0 and g["max_rel_err"] <= 1e-2
    assert g["oracle_extrapolated"] is True and g["tops"] > 0 and g["oracle_threads"] >= 1
