"""Python binding of libsq (``include/sq.h``): the same entry points, argument marshalling only.

Every step of the smoothed W8A8 linear runs in libsq's CUDA kernels. This module only checks
tensor placement / dtype, allocates outputs with PyTorch when the caller does not pass them, and
forwards raw device pointers, sizes and the current CUDA stream. Importing it fails (ImportError)
when ``libsq.so`` has not been built: there is no fallback path.

With the environment variable ``SQ_CHECKED=1`` set at import, the binding loads
``libsq_checked.so`` instead: the same kernels built with device-side bounds checks, which record
SQ_ERR_BOUNDS in the status word (read by ``sq_device_status``) and skip the access, never fault.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "SQError", "lib", "sq_calibrate_absmax", "sq_calibrate_absmax_pair", "sq_compute_scales", "sq_smooth_quantize_weight",
    "sq_rmsnorm_smooth_quant", "sq_w8a8_linear", "sq_w8a8_linear_workspace_size", "sq_device_status",
    "sq_set_wait_timeout_ns", "sq_selftest_wait_timeout", "sq_selftest_bounds_check", "sq_set_gemm_cta_pair",
    "sq_static_scale", "sq_rmsnorm_smooth_quant_static", "sq_fold_into_prev_linear", "sq_fold_into_w_scale",
    "sq_smooth_quantize_weight_fp8", "sq_rmsnorm_smooth_quant_fp8", "sq_w8a8_linear_fp8", "sq_calibrate_absmax_layernorm", "sq_fold_layernorm_bias",
    "sq_layernorm_smooth_quant", "sq_status_string", "sq_last_error",
    "sq_version", "LIB_PATH", "EXPORTS", "CHECKED",
]

CHECKED = os.environ.get("SQ_CHECKED", "0") not in ("", "0")
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libsq_checked.so" if CHECKED else "libsq.so")

SQ_OK = 0
STATUS_NAMES = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED", 3: "SQ_ERR_MISALIGNED",
                4: "SQ_ERR_ARCH", 5: "SQ_ERR_CUDA", 6: "SQ_ERR_TIMEOUT", 7: "SQ_ERR_BOUNDS"}

_p, _i64, _f, _i, _sz, _u64 = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int,
                               ctypes.c_size_t, ctypes.c_uint64)

# name -> (restype, argtypes); mirrors include/sq.h
EXPORTS = {
    "sq_status_string": (ctypes.c_char_p, [_i]),
    "sq_last_error": (ctypes.c_char_p, []),
    "sq_version": (ctypes.c_char_p, []),
    "sq_calibrate_absmax": (_i, [_p, _i64, _i64, _i64, _p, _f, _p, _i, _p]),
    "sq_calibrate_absmax_pair": (_i, [_p, _i64, _i64, _i64, _p, _f, _p, _p, _i64, _i64, _p, _i, _p]),
    "sq_compute_scales": (_i, [_p, _p, _i64, _f, _p, _p, _p, _p]),
    "sq_smooth_quantize_weight": (_i, [_p, _i64, _i64, _p, _p, _p, _p]),
    "sq_rmsnorm_smooth_quant": (_i, [_p, _i64, _i64, _p, _f, _i, _p, _p, _p]),
    "sq_w8a8_linear": (_i, [_p, _p, _i64, _p, _p, _i64, _i64, _p, _p, _p, _p, _sz, _p]),
    "sq_w8a8_linear_workspace_size": (_sz, [_i64, _i64, _i64]),
    "sq_device_status": (_i, [_p]),
    "sq_set_wait_timeout_ns": (_i, [_u64]),
    "sq_selftest_wait_timeout": (_i, [_p]),
    "sq_selftest_bounds_check": (_i, [_p]),
    "sq_set_gemm_cta_pair": (_i, [_i]),
    "sq_static_scale": (_i, [_p, _p, _i64, _p, _p]),
    "sq_rmsnorm_smooth_quant_static": (_i, [_p, _i64, _i64, _p, _f, _i, _p, _p, _p, _p]),
    "sq_fold_into_prev_linear": (_i, [_p, _p, _i64, _i64, _p, _p, _p, _p]),
    "sq_fold_into_w_scale": (_i, [_p, _i64, _p, _p, _p]),
    "sq_smooth_quantize_weight_fp8": (_i, [_p, _i64, _i64, _p, _p, _p, _p]),
    "sq_rmsnorm_smooth_quant_fp8": (_i, [_p, _i64, _i64, _p, _f, _i, _p, _p, _p]),
    "sq_w8a8_linear_fp8": (_i, [_p, _p, _i64, _p, _p, _i64, _i64, _p, _p, _p, _p, ctypes.c_size_t, _p]),
    "sq_calibrate_absmax_layernorm": (_i, [_p, _i64, _i64, _i64, _p, _p, _f, _p, _i, _p]),
    "sq_fold_layernorm_bias": (_i, [_p, _p, _i64, _p, _p]),
    "sq_layernorm_smooth_quant": (_i, [_p, _i64, _i64, _p, _p, _f, _p, _p, _p]),
}


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not found at {LIB_PATH}; build it with "
                          "`python -m post_quantization_calib_b200.build"
                          f"{' --checked' if CHECKED else ''}` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in EXPORTS.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


_lib = _load()


def lib() -> ctypes.CDLL:
    """The loaded libsq shared library (raw C entry points)."""
    return _lib


class SQError(RuntimeError):
    """A libsq call returned a status other than SQ_OK."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        msg = _lib.sq_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)}: {msg}")


def _check(st: int, where: str) -> None:
    if st != SQ_OK:
        raise SQError(st, where)


def sq_status_string(status: int) -> str:
    return _lib.sq_status_string(int(status)).decode()


def sq_last_error() -> str:
    return _lib.sq_last_error().decode(errors="replace")


def sq_version() -> str:
    return _lib.sq_version().decode()


# The current device's current stream as a raw handle. torch.cuda.current_stream() builds a Stream
# object per call (about 3 us of host time, as much as the C call itself); the two C-level lookups below
# return the same handle in about 0.1 us.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream) -> Optional[int]:
    if stream is None:
        if _raw_stream is not None and _cur_device is not None:
            return _raw_stream(_cur_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, contiguous: bool = True) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device})")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def sq_calibrate_absmax(a: torch.Tensor, norm_gamma: Optional[torch.Tensor] = None, eps: float = 1e-6,
                        amax: Optional[torch.Tensor] = None, accumulate: bool = False, stream=None) -> torch.Tensor:
    """Per-column abs-max of bf16 ``a[rows, cols]`` (rows may be strided); see sq.h."""
    _dev(a, "a", torch.bfloat16, contiguous=False)
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("a must be 2-D with unit column stride")
    rows, cols = a.shape
    if amax is None:
        amax = torch.empty(cols, dtype=torch.float32, device=a.device)
        accumulate = False
    _dev(amax, "amax", torch.float32)
    if norm_gamma is not None:
        _dev(norm_gamma, "norm_gamma", torch.float32)
    ld = a.stride(0) if a.stride(0) >= cols else cols
    _check(_lib.sq_calibrate_absmax(_ptr(a), rows, cols, ld, _ptr(norm_gamma),
                                    float(eps), _ptr(amax), int(bool(accumulate)), _stream(stream)),
           "sq_calibrate_absmax")
    return amax


def sq_calibrate_absmax_pair(a: torch.Tensor, w: torch.Tensor, norm_gamma: Optional[torch.Tensor] = None,
                             eps: float = 1e-6, amax: Optional[torch.Tensor] = None,
                             amax_w: Optional[torch.Tensor] = None, accumulate: bool = False,
                             stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-column abs-max of bf16 ``a`` (its RMSNorm output with ``norm_gamma``) and of bf16 ``w`` in
    one call; see sq.h. Returns (amax, amax_w)."""
    for t, name in ((a, "a"), (w, "w")):
        _dev(t, name, torch.bfloat16, contiguous=False)
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(f"{name} must be 2-D with unit column stride")
    rows, cols = a.shape
    w_rows, w_cols = w.shape
    if w_cols != cols:
        raise ValueError("a and w must have the same number of columns")
    if amax is None or amax_w is None:
        accumulate = False
    if amax is None:
        amax = torch.empty(cols, dtype=torch.float32, device=a.device)
    if amax_w is None:
        amax_w = torch.empty(cols, dtype=torch.float32, device=a.device)
    _dev(amax, "amax", torch.float32)
    _dev(amax_w, "amax_w", torch.float32)
    if norm_gamma is not None:
        _dev(norm_gamma, "norm_gamma", torch.float32)
    ld = a.stride(0) if a.stride(0) >= cols else cols
    w_ld = w.stride(0) if w.stride(0) >= cols else cols
    _check(_lib.sq_calibrate_absmax_pair(_ptr(a), rows, cols, ld, _ptr(norm_gamma), float(eps), _ptr(amax),
                                         _ptr(w), w_rows, w_ld, _ptr(amax_w), int(bool(accumulate)),
                                         _stream(stream)),
           "sq_calibrate_absmax_pair")
    return amax, amax_w


def sq_compute_scales(amax_x: torch.Tensor, amax_w: torch.Tensor, alpha: float,
                      gamma: Optional[torch.Tensor] = None, s: Optional[torch.Tensor] = None,
                      fold: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Smoothing factors s and folded norm weight; see sq.h."""
    _dev(amax_x, "amax_x", torch.float32)
    _dev(amax_w, "amax_w", torch.float32)
    K = amax_x.numel()
    if amax_w.numel() != K:
        raise ValueError("amax_x and amax_w must have the same length")
    if gamma is not None:
        _dev(gamma, "gamma", torch.float32)
    s = torch.empty(K, dtype=torch.float32, device=amax_x.device) if s is None else _dev(s, "s", torch.float32)
    fold = torch.empty(K, dtype=torch.float32, device=amax_x.device) if fold is None else _dev(fold, "fold", torch.float32)
    _check(_lib.sq_compute_scales(_ptr(amax_x), _ptr(amax_w), K, float(alpha), _ptr(gamma), _ptr(s), _ptr(fold),
                                  _stream(stream)), "sq_compute_scales")
    return s, fold


def sq_smooth_quantize_weight(w: torch.Tensor, s: Optional[torch.Tensor] = None, wq: Optional[torch.Tensor] = None,
                              w_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """INT8 per-output-channel quantisation of diag(s) W (w stored [N, K]); see sq.h."""
    _dev(w, "w", torch.bfloat16)
    N, K = w.shape
    if s is not None:
        _dev(s, "s", torch.float32)
    wq = torch.empty(N, K, dtype=torch.int8, device=w.device) if wq is None else _dev(wq, "wq", torch.int8)
    w_scale = torch.empty(N, dtype=torch.float32, device=w.device) if w_scale is None else _dev(w_scale, "w_scale", torch.float32)
    _check(_lib.sq_smooth_quantize_weight(_ptr(w), N, K, _ptr(s), _ptr(wq), _ptr(w_scale), _stream(stream)),
           "sq_smooth_quantize_weight")
    return wq, w_scale


def sq_rmsnorm_smooth_quant(x: torch.Tensor, fold: torch.Tensor, eps: float = 1e-6, apply_norm: bool = True,
                            xq: Optional[torch.Tensor] = None, x_scale: Optional[torch.Tensor] = None,
                            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused RMSNorm (folded 1/s) + per-token INT8 quantisation; see sq.h."""
    _dev(x, "x", torch.bfloat16)
    _dev(fold, "fold", torch.float32)
    T, K = x.shape
    xq = torch.empty(T, K, dtype=torch.int8, device=x.device) if xq is None else _dev(xq, "xq", torch.int8)
    x_scale = torch.empty(T, dtype=torch.float32, device=x.device) if x_scale is None else _dev(x_scale, "x_scale", torch.float32)
    _check(_lib.sq_rmsnorm_smooth_quant(_ptr(x), T, K, _ptr(fold), float(eps), int(bool(apply_norm)), _ptr(xq),
                                        _ptr(x_scale), _stream(stream)), "sq_rmsnorm_smooth_quant")
    return xq, x_scale


def sq_static_scale(amax: torch.Tensor, factor: Optional[torch.Tensor] = None, scale2: Optional[torch.Tensor] = None,
                    stream=None) -> torch.Tensor:
    """Static per-tensor activation scale {delta, 127/m} from a calibration maximum; see sq.h."""
    _dev(amax, "amax", torch.float32)
    K = amax.shape[0]
    if factor is not None:
        _dev(factor, "factor", torch.float32)
    scale2 = torch.empty(2, dtype=torch.float32, device=amax.device) if scale2 is None else _dev(scale2, "scale2", torch.float32)
    _check(_lib.sq_static_scale(_ptr(amax), _ptr(factor), K, _ptr(scale2), _stream(stream)), "sq_static_scale")
    return scale2


def sq_rmsnorm_smooth_quant_static(x: torch.Tensor, fold: torch.Tensor, scale2: torch.Tensor, eps: float = 1e-6,
                                   apply_norm: bool = True, xq: Optional[torch.Tensor] = None,
                                   x_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused RMSNorm (folded 1/s) + INT8 with the static per-tensor scale; see sq.h."""
    _dev(x, "x", torch.bfloat16)
    _dev(fold, "fold", torch.float32)
    _dev(scale2, "scale2", torch.float32)
    T, K = x.shape
    xq = torch.empty(T, K, dtype=torch.int8, device=x.device) if xq is None else _dev(xq, "xq", torch.int8)
    x_scale = torch.empty(T, dtype=torch.float32, device=x.device) if x_scale is None else _dev(x_scale, "x_scale", torch.float32)
    _check(_lib.sq_rmsnorm_smooth_quant_static(_ptr(x), T, K, _ptr(fold), float(eps), int(bool(apply_norm)), _ptr(scale2),
                                               _ptr(xq), _ptr(x_scale), _stream(stream)), "sq_rmsnorm_smooth_quant_static")
    return xq, x_scale


def sq_fold_into_prev_linear(w: torch.Tensor, fold: torch.Tensor, b: Optional[torch.Tensor] = None,
                             w_out: Optional[torch.Tensor] = None, b_out: Optional[torch.Tensor] = None,
                             stream=None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Previous bf16 linear [K, Kp] with output channel j multiplied by fold[j]; see sq.h."""
    _dev(w, "w", torch.bfloat16)
    _dev(fold, "fold", torch.float32)
    K, Kp = w.shape
    w_out = torch.empty_like(w) if w_out is None else _dev(w_out, "w_out", torch.bfloat16)
    if b is not None:
        _dev(b, "b", torch.bfloat16)
        b_out = torch.empty_like(b) if b_out is None else _dev(b_out, "b_out", torch.bfloat16)
    _check(_lib.sq_fold_into_prev_linear(_ptr(w), _ptr(b), K, Kp, _ptr(fold), _ptr(w_out), _ptr(b_out) if b is not None else None,
                                         _stream(stream)), "sq_fold_into_prev_linear")
    return w_out, (b_out if b is not None else None)


def sq_fold_into_w_scale(w_scale: torch.Tensor, fold: torch.Tensor, out: Optional[torch.Tensor] = None,
                         stream=None) -> torch.Tensor:
    """INT8 previous layer: per-channel dequantisation scale times fold; see sq.h."""
    _dev(w_scale, "w_scale", torch.float32)
    _dev(fold, "fold", torch.float32)
    out = torch.empty_like(w_scale) if out is None else _dev(out, "out", torch.float32)
    _check(_lib.sq_fold_into_w_scale(_ptr(w_scale), w_scale.shape[0], _ptr(fold), _ptr(out), _stream(stream)),
           "sq_fold_into_w_scale")
    return out


def sq_calibrate_absmax_layernorm(a: torch.Tensor, gamma: torch.Tensor, beta: Optional[torch.Tensor] = None,
                                  eps: float = 1e-5, amax: Optional[torch.Tensor] = None, accumulate: bool = False,
                                  stream=None) -> torch.Tensor:
    """Per-column abs-max of LayerNorm(a) * gamma + beta (a bf16, rows may be strided); see sq.h."""
    _dev(a, "a", torch.bfloat16, contiguous=False)
    if a.dim() != 2 or a.stride(1) != 1:
        raise ValueError("a must be 2-D with unit column stride")
    rows, cols = a.shape
    if amax is None:
        amax = torch.empty(cols, dtype=torch.float32, device=a.device)
        accumulate = False
    _dev(amax, "amax", torch.float32)
    _dev(gamma, "gamma", torch.float32)
    if beta is not None:
        _dev(beta, "beta", torch.float32)
    ld = a.stride(0) if a.stride(0) >= cols else cols
    _check(_lib.sq_calibrate_absmax_layernorm(_ptr(a), rows, cols, ld, _ptr(gamma), _ptr(beta), float(eps), _ptr(amax),
                                              int(bool(accumulate)), _stream(stream)), "sq_calibrate_absmax_layernorm")
    return amax


def sq_fold_layernorm_bias(beta: torch.Tensor, s: torch.Tensor, out: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """LayerNorm bias with S^-1 folded in, beta / s; see sq.h."""
    _dev(beta, "beta", torch.float32)
    _dev(s, "s", torch.float32)
    if s.numel() != beta.numel():
        raise ValueError("beta and s must have the same length")
    out = torch.empty_like(beta) if out is None else _dev(out, "out", torch.float32)
    _check(_lib.sq_fold_layernorm_bias(_ptr(beta), _ptr(s), beta.numel(), _ptr(out), _stream(stream)),
           "sq_fold_layernorm_bias")
    return out


def sq_layernorm_smooth_quant(x: torch.Tensor, fold: torch.Tensor, beta_fold: Optional[torch.Tensor] = None,
                              eps: float = 1e-5, xq: Optional[torch.Tensor] = None,
                              x_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused LayerNorm (gamma / s, beta / s folded in) + per-token INT8 quantisation; see sq.h."""
    _dev(x, "x", torch.bfloat16)
    _dev(fold, "fold", torch.float32)
    if beta_fold is not None:
        _dev(beta_fold, "beta_fold", torch.float32)
    T, K = x.shape
    xq = torch.empty(T, K, dtype=torch.int8, device=x.device) if xq is None else _dev(xq, "xq", torch.int8)
    x_scale = torch.empty(T, dtype=torch.float32, device=x.device) if x_scale is None else _dev(x_scale, "x_scale", torch.float32)
    _check(_lib.sq_layernorm_smooth_quant(_ptr(x), T, K, _ptr(fold), _ptr(beta_fold), float(eps), _ptr(xq), _ptr(x_scale),
                                          _stream(stream)), "sq_layernorm_smooth_quant")
    return xq, x_scale


def sq_smooth_quantize_weight_fp8(w: torch.Tensor, s: Optional[torch.Tensor] = None, wq: Optional[torch.Tensor] = None,
                                  w_scale: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """diag(s)*W quantised to FP8 E4M3 (uint8 codes) per output channel; see sq.h."""
    _dev(w, "w", torch.bfloat16)
    N, K = w.shape
    if s is not None:
        _dev(s, "s", torch.float32)
    wq = torch.empty(N, K, dtype=torch.uint8, device=w.device) if wq is None else _dev(wq, "wq", torch.uint8)
    w_scale = torch.empty(N, dtype=torch.float32, device=w.device) if w_scale is None else _dev(w_scale, "w_scale", torch.float32)
    _check(_lib.sq_smooth_quantize_weight_fp8(_ptr(w), N, K, _ptr(s), _ptr(wq), _ptr(w_scale), _stream(stream)),
           "sq_smooth_quantize_weight_fp8")
    return wq, w_scale


def sq_rmsnorm_smooth_quant_fp8(x: torch.Tensor, fold: torch.Tensor, eps: float = 1e-6, apply_norm: bool = True,
                                xq: Optional[torch.Tensor] = None, x_scale: Optional[torch.Tensor] = None,
                                stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Fused RMSNorm (folded 1/s) + per-token FP8 E4M3 (uint8 codes); see sq.h."""
    _dev(x, "x", torch.bfloat16)
    _dev(fold, "fold", torch.float32)
    T, K = x.shape
    xq = torch.empty(T, K, dtype=torch.uint8, device=x.device) if xq is None else _dev(xq, "xq", torch.uint8)
    x_scale = torch.empty(T, dtype=torch.float32, device=x.device) if x_scale is None else _dev(x_scale, "x_scale", torch.float32)
    _check(_lib.sq_rmsnorm_smooth_quant_fp8(_ptr(x), T, K, _ptr(fold), float(eps), int(bool(apply_norm)), _ptr(xq),
                                            _ptr(x_scale), _stream(stream)), "sq_rmsnorm_smooth_quant_fp8")
    return xq, x_scale


def sq_w8a8_linear_fp8(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                       bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                       acc_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """FP8 E4M3 GEMM (binary32 accumulation) with the dequant epilogue -> bf16 [T, N]; see sq.h."""
    _dev(xq, "xq", torch.uint8)
    _dev(x_scale, "x_scale", torch.float32)
    _dev(wq, "wq", torch.uint8)
    _dev(w_scale, "w_scale", torch.float32)
    T, K = xq.shape
    N, K2 = wq.shape
    if K2 != K:
        raise ValueError(f"inner sizes differ: xq has K={K}, wq has K={K2}")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=xq.device) if y is None else _dev(y, "y", torch.bfloat16)
    if acc_out is not None:
        _dev(acc_out, "acc_out", torch.float32)
    _check(_lib.sq_w8a8_linear_fp8(_ptr(xq), _ptr(x_scale), T, _ptr(wq), _ptr(w_scale), N, K, _ptr(bias), _ptr(y),
                                   _ptr(acc_out), None, 0, _stream(stream)), "sq_w8a8_linear_fp8")
    return y


def sq_w8a8_linear(xq: torch.Tensor, x_scale: torch.Tensor, wq: torch.Tensor, w_scale: torch.Tensor,
                   bias: Optional[torch.Tensor] = None, y: Optional[torch.Tensor] = None,
                   acc_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """INT8 GEMM with fused dequant epilogue -> bf16 [T, N]; see sq.h."""
    _dev(xq, "xq", torch.int8)
    _dev(x_scale, "x_scale", torch.float32)
    _dev(wq, "wq", torch.int8)
    _dev(w_scale, "w_scale", torch.float32)
    T, K = xq.shape
    N, K2 = wq.shape
    if K2 != K:
        raise ValueError(f"inner sizes differ: xq has K={K}, wq has K={K2}")
    if bias is not None:
        _dev(bias, "bias", torch.bfloat16)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=xq.device) if y is None else _dev(y, "y", torch.bfloat16)
    if acc_out is not None:
        _dev(acc_out, "acc_out", torch.int32)
    _check(_lib.sq_w8a8_linear(_ptr(xq), _ptr(x_scale), T, _ptr(wq), _ptr(w_scale), N, K, _ptr(bias), _ptr(y),
                               _ptr(acc_out), None, 0, _stream(stream)), "sq_w8a8_linear")
    return y


def sq_w8a8_linear_workspace_size(T: int, N: int, K: int) -> int:
    return int(_lib.sq_w8a8_linear_workspace_size(T, N, K))


def sq_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word; 0 = SQ_OK."""
    return int(_lib.sq_device_status(_stream(stream)))


def sq_set_wait_timeout_ns(ns: int) -> None:
    _check(_lib.sq_set_wait_timeout_ns(int(ns)), "sq_set_wait_timeout_ns")


def sq_set_gemm_cta_pair(enable: bool) -> None:
    """Selects the GEMM form for later calls: CTA pairs (True) or one SM per tile (False, default)."""
    _check(_lib.sq_set_gemm_cta_pair(1 if enable else 0), "sq_set_gemm_cta_pair")


def sq_selftest_wait_timeout(stream=None) -> None:
    _check(_lib.sq_selftest_wait_timeout(_stream(stream)), "sq_selftest_wait_timeout")


def sq_selftest_bounds_check(stream=None) -> None:
    """Launch the failing bounds check of libsq_checked.so (SQ_ERR_UNSUPPORTED in libsq.so)."""
    _check(_lib.sq_selftest_bounds_check(_stream(stream)), "sq_selftest_bounds_check")
