"""GPU: the checked library (libsq_checked.so), the kernels built with device-side bounds checks.

Each check guards one access: the copies of a row group into its ring slot, the row kernels' code,
scale and abs-max stores, the column bound that a FULL geometry takes for granted, the GEMM's TMA
coordinates and its accumulator stores. A failed check records SQ_ERR_BOUNDS in the device status
word and skips the access, so an index error surfaces as a status instead of a fault. The checked
library is loaded in child processes (SQ_CHECKED=1), since this process holds the product library.
"""
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# parity tests that reach every row-kernel mode and geometry, every GEMM form and the folds
SUBSET = " or ".join([
    "single_linear_full", "block_prefill_groups", "edge_shapes", "extreme_codes", "absmax_strided", "absmax_pair",
    "cta_pair_gemm", "decode_form_buckets", "static_scale_path", "fold_into_prev_linear", "fp8_path",
    "layernorm_fold_path", "layer_object", "layer_fold_into_previous", "quantisers_over_few_rows",
])

SELFTEST = """
from post_quantization_calib_b200 import sq
assert sq.CHECKED and sq.LIB_PATH.endswith("libsq_checked.so"), sq.LIB_PATH
assert sq.sq_device_status() == 0
sq.sq_selftest_bounds_check()
st = sq.sq_device_status()
assert st == 7, sq.sq_status_string(st)          # SQ_ERR_BOUNDS, recorded by the kernel
assert sq.sq_device_status() == 0                # reading cleared it
import torch
xq = torch.ones(128, 256, dtype=torch.int8, device="cuda")
y = sq.sq_w8a8_linear(xq, torch.ones(128, device="cuda"), xq.clone(), torch.ones(128, device="cuda"))
assert sq.sq_device_status() == 0 and bool(torch.all(y.float() == 256.0))
print("checked-selftest-ok")
"""


def child_env():
    env = dict(os.environ)
    env["SQ_CHECKED"] = "1"
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    return env


@pytest.fixture(scope="module")
def checked_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from post_quantization_calib_b200 import build
    return build.build(checked=True)


def test_product_library_has_no_checks():
    from post_quantization_calib_b200 import build
    build.build()
    from post_quantization_calib_b200 import sq
    assert not sq.CHECKED
    with pytest.raises(sq.SQError) as e:
        sq.sq_selftest_bounds_check()
    assert e.value.status == 2                   # SQ_ERR_UNSUPPORTED: nothing launched


def test_failed_check_is_recorded_and_skipped(checked_lib):
    r = subprocess.run([sys.executable, "-c", SELFTEST], cwd=ROOT, env=child_env(),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "checked-selftest-ok" in r.stdout, r.stdout[-2000:] + r.stderr[-2000:]


def test_parity_subset_passes_with_every_check(checked_lib):
    cmd = [sys.executable, "-m", "pytest", os.path.join("tests", "test_parity_gpu.py"), "-m", "gpu", "-x", "-q",
           "-p", "no:cacheprovider", "-k", SUBSET]
    r = subprocess.run(cmd, cwd=ROOT, env=child_env(), capture_output=True, text=True, timeout=1800)
    tail = r.stdout[-3000:] + r.stderr[-2000:]
    assert r.returncode == 0, tail
    assert " passed" in r.stdout and " failed" not in r.stdout, tail
