"""libsq's C ABI on a host without a GPU: the library loads, exports every function include/sq.h
declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq.h")

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_MISALIGNED, SQ_ERR_ARCH, SQ_ERR_CUDA, SQ_ERR_TIMEOUT, SQ_ERR_BOUNDS = range(8)


@pytest.fixture(scope="module")
def sqmod():
    from post_quantization_calib_b200 import build
    build.build()
    from post_quantization_calib_b200 import sq
    return sq


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_five_calls():
    names = declared_functions()
    for n in ("sq_calibrate_absmax", "sq_compute_scales", "sq_smooth_quantize_weight",
              "sq_rmsnorm_smooth_quant", "sq_w8a8_linear"):
        assert n in names


def test_library_exports_every_declared_symbol(sqmod):
    names = declared_functions()
    L = sqmod.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in sq.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", sqmod.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sq_[a-z0-9_]+)", out))
    assert set(names) <= exported
    # the binding wraps exactly the declared set
    assert set(sqmod.EXPORTS) == set(names)


def test_checked_library_exports_the_same_symbols(sqmod):
    """libsq_checked.so (device bounds checks compiled in) exports the same C ABI as libsq.so."""
    from post_quantization_calib_b200 import build
    path = build.build(checked=True)
    assert path.endswith("libsq_checked.so") and path != sqmod.LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (sq_[a-z0-9_]+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings(sqmod):
    names = [sqmod.sq_status_string(i) for i in range(8)]
    assert names == ["SQ_OK", "SQ_ERR_INVALID_ARG", "SQ_ERR_UNSUPPORTED", "SQ_ERR_MISALIGNED",
                     "SQ_ERR_ARCH", "SQ_ERR_CUDA", "SQ_ERR_TIMEOUT", "SQ_ERR_BOUNDS"]
    assert all(sqmod.STATUS_NAMES[i] == names[i] for i in range(8))
    assert sqmod.sq_status_string(99) == "SQ_ERR_UNKNOWN"
    assert "sm_100a" in sqmod.sq_version()


def test_workspace_size_is_zero(sqmod):
    assert sqmod.sq_w8a8_linear_workspace_size(8192, 4096, 4096) == 0


def test_gemm_form_setter_checks_its_argument(sqmod):
    L = sqmod._lib
    assert L.sq_set_gemm_cta_pair(2) == 1            # SQ_ERR_INVALID_ARG
    assert L.sq_set_gemm_cta_pair(-1) == 1
    assert L.sq_set_gemm_cta_pair(1) == 0
    assert L.sq_set_gemm_cta_pair(0) == 0            # back to the default


# Argument checks run before any CUDA call, so they behave the same with or without a GPU.
FAKE = 0x10000   # a 16-byte aligned address that is never dereferenced


def test_absmax_argument_checks(sqmod):
    L = sqmod.lib()
    assert L.sq_calibrate_absmax(FAKE, 4, 64, 64, None, 1e-6, None, 0, None) == SQ_ERR_INVALID_ARG
    assert L.sq_calibrate_absmax(FAKE, -1, 64, 64, None, 1e-6, FAKE, 0, None) == SQ_ERR_INVALID_ARG
    assert L.sq_calibrate_absmax(FAKE, 4, 64, 32, None, 1e-6, FAKE, 0, None) == SQ_ERR_INVALID_ARG
    assert L.sq_calibrate_absmax(FAKE, 4, 60, 64, None, 1e-6, FAKE, 0, None) == SQ_ERR_MISALIGNED
    assert L.sq_calibrate_absmax(FAKE + 8, 4, 64, 64, None, 1e-6, FAKE, 0, None) == SQ_ERR_MISALIGNED
    assert L.sq_calibrate_absmax(FAKE, 4, 32768, 32768, FAKE, 1e-6, FAKE, 0, None) == SQ_ERR_UNSUPPORTED
    assert L.sq_calibrate_absmax(FAKE, 4, 16392, 16392, None, 1e-6, FAKE, 0, None) == SQ_ERR_UNSUPPORTED
    assert "cols" in sqmod.sq_last_error()


def test_scales_argument_checks(sqmod):
    L = sqmod.lib()
    assert L.sq_compute_scales(FAKE, FAKE, 16, 1.5, None, FAKE, None, None) == SQ_ERR_INVALID_ARG
    assert L.sq_compute_scales(FAKE, FAKE, 16, -0.1, None, FAKE, None, None) == SQ_ERR_INVALID_ARG
    assert L.sq_compute_scales(FAKE, FAKE, 16, float("nan"), None, FAKE, None, None) == SQ_ERR_INVALID_ARG
    assert L.sq_compute_scales(FAKE, None, 16, 0.5, None, FAKE, None, None) == SQ_ERR_INVALID_ARG
    assert L.sq_compute_scales(FAKE, FAKE, 0, 0.5, None, FAKE, None, None) == SQ_ERR_INVALID_ARG
    assert L.sq_compute_scales(FAKE + 2, FAKE, 16, 0.5, None, FAKE, None, None) == SQ_ERR_MISALIGNED


def test_static_scale_argument_checks(sqmod):
    L = sqmod.lib()
    assert L.sq_static_scale(None, None, 16, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_static_scale(FAKE, None, 0, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_static_scale(FAKE + 2, None, 16, FAKE, None) == SQ_ERR_MISALIGNED
    q = L.sq_rmsnorm_smooth_quant_static
    assert q(FAKE, 4, 64, FAKE, 1e-6, 1, None, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG       # no scale2
    assert q(FAKE, 4, 12, FAKE, 1e-6, 1, FAKE, FAKE, FAKE, None) == SQ_ERR_MISALIGNED        # K % 8
    assert q(FAKE, 4, 32768, FAKE, 1e-6, 1, FAKE, FAKE, FAKE, None) == SQ_ERR_UNSUPPORTED
    assert q(FAKE + 8, 4, 64, FAKE, 1e-6, 1, FAKE, FAKE, FAKE, None) == SQ_ERR_MISALIGNED    # x alignment


def test_fold_argument_checks(sqmod):
    L = sqmod.lib()
    f = L.sq_fold_into_prev_linear
    assert f(FAKE, None, 4, 64, None, FAKE, None, None) == SQ_ERR_INVALID_ARG      # no fold
    assert f(FAKE, FAKE, 4, 64, FAKE, FAKE, None, None) == SQ_ERR_INVALID_ARG      # bias without b_out
    assert f(FAKE, None, 4, 12, FAKE, FAKE, None, None) == SQ_ERR_MISALIGNED       # Kp % 8
    assert f(FAKE + 8, None, 4, 64, FAKE, FAKE, None, None) == SQ_ERR_MISALIGNED   # w alignment
    assert L.sq_fold_into_w_scale(FAKE, 0, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_fold_into_w_scale(FAKE + 2, 8, FAKE, FAKE, None) == SQ_ERR_MISALIGNED


def test_layernorm_argument_checks(sqmod):
    L = sqmod.lib()
    c = L.sq_calibrate_absmax_layernorm
    assert c(FAKE, 4, 64, 64, None, None, 1e-5, FAKE, 0, None) == SQ_ERR_INVALID_ARG       # no gamma
    assert c(FAKE, 4, 64, 32, FAKE, None, 1e-5, FAKE, 0, None) == SQ_ERR_INVALID_ARG       # ld < cols
    assert c(FAKE, 4, 12, 12, FAKE, None, 1e-5, FAKE, 0, None) == SQ_ERR_MISALIGNED        # cols % 8
    assert c(FAKE, 4, 64, 64, FAKE, FAKE + 4, 1e-5, FAKE, 0, None) == SQ_ERR_MISALIGNED    # beta alignment
    assert c(FAKE, 4, 32768, 32768, FAKE, None, 1e-5, FAKE, 0, None) == SQ_ERR_UNSUPPORTED
    assert L.sq_fold_layernorm_bias(FAKE, None, 8, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_fold_layernorm_bias(FAKE, FAKE, 0, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_fold_layernorm_bias(FAKE + 2, FAKE, 8, FAKE, None) == SQ_ERR_MISALIGNED
    q = L.sq_layernorm_smooth_quant
    assert q(FAKE, 4, 64, None, None, 1e-5, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG         # no fold
    assert q(FAKE, 4, 64, FAKE, FAKE + 4, 1e-5, FAKE, FAKE, None) == SQ_ERR_MISALIGNED      # beta_fold alignment
    assert q(FAKE, 4, 32768, FAKE, None, 1e-5, FAKE, FAKE, None) == SQ_ERR_UNSUPPORTED
    assert q(FAKE, -1, 64, FAKE, None, 1e-5, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG


def test_absmax_pair_argument_checks(sqmod):
    c = sqmod.lib().sq_calibrate_absmax_pair
    G = FAKE + 4096
    #        a     rows cols ld   gamma eps   amax  w     wrows wld  amax_w acc stream
    assert c(FAKE, 4, 64, 64, None, 1e-6, None, FAKE, 4, 64, G, 0, None) == SQ_ERR_INVALID_ARG     # amax NULL
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, 4, 64, None, 0, None) == SQ_ERR_INVALID_ARG     # amax_w NULL
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, 4, 64, G, 0, None) == SQ_ERR_INVALID_ARG        # same array
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, 4, 64, G + 4 * 63, 0, None) == SQ_ERR_INVALID_ARG  # overlap
    assert c(FAKE, 4, 64, 64, None, 1e-6, G + 4 * 63, FAKE, 4, 64, G, 0, None) == SQ_ERR_INVALID_ARG  # overlap
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, 4, 32, G + 256, 0, None) == SQ_ERR_INVALID_ARG  # w_ld < cols
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, None, 4, 64, G + 256, 0, None) == SQ_ERR_INVALID_ARG  # w NULL with rows
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, -1, 64, G + 256, 0, None) == SQ_ERR_INVALID_ARG # w_rows < 0
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE + 2, 4, 64, G + 256, 0, None) == SQ_ERR_MISALIGNED
    assert c(FAKE, 4, 64, 64, FAKE + 4, 1e-6, G, FAKE, 4, 64, G + 256, 0, None) == SQ_ERR_MISALIGNED  # gamma
    assert c(FAKE, 4, 64, 64, None, 1e-6, G, FAKE, 4, 68, G + 256, 0, None) == SQ_ERR_MISALIGNED   # w_ld % 8
    assert c(FAKE, 4, 32768, 32768, None, 1e-6, G, FAKE, 4, 32768, G + 256, 0, None) == SQ_ERR_UNSUPPORTED


def test_fp8_argument_checks(sqmod):
    L = sqmod.lib()
    assert L.sq_smooth_quantize_weight_fp8(FAKE, 4, 12, None, FAKE, FAKE, None) == SQ_ERR_MISALIGNED
    assert L.sq_smooth_quantize_weight_fp8(FAKE, 4, 32768, None, FAKE, FAKE, None) == SQ_ERR_UNSUPPORTED
    assert L.sq_rmsnorm_smooth_quant_fp8(FAKE, 4, 64, None, 1e-6, 1, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG
    g = L.sq_w8a8_linear_fp8
    assert g(FAKE, FAKE, 4, FAKE, FAKE, 4, 64, None, FAKE, None, None, 0, None) == SQ_ERR_INVALID_ARG   # N < 8
    assert g(FAKE, FAKE, 4, FAKE, FAKE, 12, 64, None, FAKE, None, None, 0, None) == SQ_ERR_MISALIGNED   # N % 8
    assert g(FAKE, FAKE, 4, None, FAKE, 16, 64, None, FAKE, None, None, 0, None) == SQ_ERR_INVALID_ARG  # no wq


def test_quant_argument_checks(sqmod):
    L = sqmod.lib()
    assert L.sq_smooth_quantize_weight(FAKE, 4, 12, None, FAKE, FAKE, None) == SQ_ERR_MISALIGNED
    assert L.sq_smooth_quantize_weight(FAKE, 4, 32768, None, FAKE, FAKE, None) == SQ_ERR_UNSUPPORTED
    assert L.sq_smooth_quantize_weight(None, 4, 64, None, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_rmsnorm_smooth_quant(FAKE, 4, 64, None, 1e-6, 1, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG
    assert L.sq_rmsnorm_smooth_quant(FAKE, 4, 64, FAKE, 1e-6, 1, FAKE + 4, FAKE, None) == SQ_ERR_MISALIGNED
    assert L.sq_rmsnorm_smooth_quant(FAKE, -2, 64, FAKE, 1e-6, 1, FAKE, FAKE, None) == SQ_ERR_INVALID_ARG


def test_linear_argument_checks(sqmod):
    L = sqmod.lib()
    ok = dict(xq=FAKE, xs=FAKE, T=16, wq=FAKE, ws=FAKE, N=64, K=64, bias=None, y=FAKE, acc=None)

    def call(**kw):
        a = {**ok, **kw}
        return L.sq_w8a8_linear(a["xq"], a["xs"], a["T"], a["wq"], a["ws"], a["N"], a["K"], a["bias"], a["y"],
                                a["acc"], None, 0, None)

    assert call(N=4) == SQ_ERR_INVALID_ARG
    assert call(K=8) == SQ_ERR_INVALID_ARG
    assert call(N=68) == SQ_ERR_MISALIGNED
    assert call(K=72) == SQ_ERR_MISALIGNED
    assert call(wq=None) == SQ_ERR_INVALID_ARG
    assert call(y=None) == SQ_ERR_INVALID_ARG
    assert call(xq=FAKE + 8) == SQ_ERR_MISALIGNED
    assert call(acc=FAKE + 4) == SQ_ERR_MISALIGNED
    assert call(bias=FAKE + 2) == SQ_ERR_MISALIGNED
    assert call(K=262144) == SQ_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_device_reports_cuda_error(sqmod):
    L = sqmod.lib()
    st = L.sq_compute_scales(FAKE, FAKE, 16, 0.5, None, FAKE, None, None)
    assert st == SQ_ERR_CUDA
    assert "cudaGetDevice" in sqmod.sq_last_error()


def test_binding_rejects_host_tensors(sqmod):
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sqmod.sq_rmsnorm_smooth_quant(x, torch.ones(64))
    with pytest.raises(ValueError):
        sqmod.sq_calibrate_absmax(x)


def test_layer_object_rejects_unsupported_combinations(sqmod):
    from post_quantization_calib_b200.layer import SmoothedW8A8Linear
    w = [torch.zeros(16, 64, dtype=torch.bfloat16)]
    g = torch.ones(64)
    with pytest.raises(ValueError):
        SmoothedW8A8Linear(w, 0.5, gamma=g, scheme="int4")
    with pytest.raises(ValueError):
        SmoothedW8A8Linear(w, 0.5, gamma=g, norm="layer", scheme="fp8")        # LayerNorm: INT8 only
    with pytest.raises(ValueError):
        SmoothedW8A8Linear(w, 0.5, gamma=None, norm="rms")                     # a norm needs gamma
    with pytest.raises(ValueError):
        SmoothedW8A8Linear(w, 0.5, gamma=g, beta=g, norm="rms")                # beta is a LayerNorm's
    layer = SmoothedW8A8Linear(w, 0.5, gamma=g, norm="layer", beta=g)
    assert layer.eps == 1e-5 and layer.norm == "layer" and layer.wq.dtype == torch.int8
    assert SmoothedW8A8Linear(w, 0.5, scheme="fp8").wq.dtype == torch.uint8
