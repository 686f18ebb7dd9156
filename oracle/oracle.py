"""numpy-facing wrappers around the C oracle (``sq_oracle.c``).

Test infrastructure. bf16 tensors travel as ``np.uint16`` bit patterns; every array must be
C-contiguous. Each wrapper names the page passage its C function follows (see the C source).
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from . import build as _build

__all__ = [
    "calibrate_absmax", "compute_scales", "smooth_quantize_weight", "rmsnorm_smooth_quant",
    "static_scale", "rmsnorm_smooth_quant_static", "fold_into_prev_linear", "fold_into_w_scale",
    "e4m3_encode", "e4m3_decode", "smooth_quantize_weight_f8", "rmsnorm_smooth_quant_f8", "gemm_f8", "dequant_f32",
    "w8a8_linear_f8", "calibrate_absmax_layernorm", "fold_layernorm_bias", "layernorm_smooth_quant",
    "gemm_s8", "dequant", "w8a8_linear", "f32_to_bf16", "bf16_to_f32", "set_threads", "lib",
]

_lock = threading.Lock()
_lib = None

_p = ctypes.c_void_p
_i64 = ctypes.c_int64


def lib() -> ctypes.CDLL:
    """Load (building first if needed) the oracle shared library."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.build()
            L = ctypes.CDLL(path)
            L.orc_calibrate_absmax.argtypes = [_p, _i64, _i64, _i64, _p, ctypes.c_float, _p, ctypes.c_int]
            L.orc_compute_scales.argtypes = [_p, _p, _i64, ctypes.c_float, _p, _p, _p]
            L.orc_smooth_quantize_weight.argtypes = [_p, _i64, _i64, _p, _p, _p, _p]
            L.orc_rmsnorm_smooth_quant.argtypes = [_p, _i64, _i64, _p, ctypes.c_float, ctypes.c_int, _p, _p, _p]
            L.orc_static_scale.argtypes = [_p, _i64, _p]
            L.orc_rmsnorm_smooth_quant_static.argtypes = [_p, _i64, _i64, _p, ctypes.c_float, ctypes.c_int, _p, _p, _p]
            L.orc_fold_into_prev_linear.argtypes = [_p, _p, _i64, _i64, _p, _p, _p]
            L.orc_fold_into_w_scale.argtypes = [_p, _i64, _p, _p]
            L.orc_e4m3_encode.argtypes = [ctypes.c_float]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_decode.restype = ctypes.c_float
            L.orc_smooth_quantize_weight_f8.argtypes = [_p, _i64, _i64, _p, _p, _p, _p]
            L.orc_rmsnorm_smooth_quant_f8.argtypes = [_p, _i64, _i64, _p, ctypes.c_float, ctypes.c_int, _p, _p, _p]
            L.orc_gemm_f8.argtypes = [_p, _i64, _p, _i64, _i64, _p, _i64, _p, _i64, _p]
            L.orc_dequant_f32.argtypes = [_p, _p, _p, _p, _p, _i64, _p, _i64, _p]
            L.orc_calibrate_absmax_layernorm.argtypes = [_p, _i64, _i64, _i64, _p, _p, ctypes.c_float, _p, ctypes.c_int, _p]
            L.orc_fold_layernorm_bias.argtypes = [_p, _p, _i64, _p]
            L.orc_layernorm_smooth_quant.argtypes = [_p, _i64, _i64, _p, _p, ctypes.c_float, _p, _p, _p]
            L.orc_gemm_s8.argtypes = [_p, _i64, _p, _i64, _i64, _p, _i64, _p, _i64, _p]
            L.orc_dequant.argtypes = [_p, _p, _p, _p, _p, _i64, _p, _i64, _p]
            L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
            L.orc_f32_to_bf16.restype = ctypes.c_uint16
            L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.orc_bf16_to_f32.restype = ctypes.c_float
            _lib = L
    return _lib


def set_threads(n: int) -> None:
    """Set the OpenMP thread count used by the oracle's GEMM."""
    os.environ["OMP_NUM_THREADS"] = str(int(n))
    try:
        omp = ctypes.CDLL("libgomp.so.1")
        omp.omp_set_num_threads(ctypes.c_int(int(n)))
    except OSError:
        pass


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _need(a, dtype, name):
    if a.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {a.dtype}")
    return np.ascontiguousarray(a)


def calibrate_absmax(a, ld=None, norm_gamma=None, eps=1e-6, amax=None, accumulate=False):
    """Per-column abs-max of bf16 ``a[rows, cols]`` (optionally of its RMSNorm output).

    [MIGRATE] section 3; [TAMING] "System Architecture". Returns ``amax`` (float32 [cols]).
    """
    a = _need(a, np.uint16, "a")
    rows, cols = a.shape
    ld = cols if ld is None else ld
    if amax is None:
        amax = np.zeros(cols, np.float32)
    g = None if norm_gamma is None else _need(np.asarray(norm_gamma), np.float32, "norm_gamma")
    lib().orc_calibrate_absmax(_ptr(a), rows, cols, ld, _ptr(g), float(eps), _ptr(amax), int(bool(accumulate)))
    return amax


def compute_scales(amax_x, amax_w, alpha, gamma=None):
    """Smoothing factors s and the folded norm weight; [MIGRATE] section 3. Returns (s, fold)."""
    ax = _need(amax_x, np.float32, "amax_x")
    aw = _need(amax_w, np.float32, "amax_w")
    K = ax.shape[0]
    s = np.empty(K, np.float32)
    fold = np.empty(K, np.float32)
    g = None if gamma is None else _need(np.asarray(gamma), np.float32, "gamma")
    lib().orc_compute_scales(_ptr(ax), _ptr(aw), K, float(alpha), _ptr(g), _ptr(s), _ptr(fold))
    return s, fold


def smooth_quantize_weight(w, s=None):
    """diag(s)*W then INT8 per output row; [MIGRATE] sections 2 and 7. Returns (wq, w_scale)."""
    w = _need(w, np.uint16, "w")
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    ws = np.empty(N, np.float32)
    work = np.empty(K, np.float32)
    sv = None if s is None else _need(s, np.float32, "s")
    lib().orc_smooth_quantize_weight(_ptr(w), N, K, _ptr(sv), _ptr(wq), _ptr(ws), _ptr(work))
    return wq, ws


def rmsnorm_smooth_quant(x, fold, eps=1e-6, apply_norm=True):
    """(RMSNorm with folded weight, or x*fold) then per-token INT8. Returns (xq, x_scale)."""
    x = _need(x, np.uint16, "x")
    T, K = x.shape
    f = _need(fold, np.float32, "fold")
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    work = np.empty(K, np.float32)
    lib().orc_rmsnorm_smooth_quant(_ptr(x), T, K, _ptr(f), float(eps), int(bool(apply_norm)),
                                   _ptr(xq), _ptr(xs), _ptr(work))
    return xq, xs


def static_scale(amax_y):
    """Static per-tensor scale from the calibration maximum of the smoothed activation
    ([W8A8] "One layer, measured"). Returns float32 [2] = (delta, 127 / m)."""
    a = _need(amax_y, np.float32, "amax_y")
    out = np.empty(2, np.float32)
    lib().orc_static_scale(_ptr(a), a.shape[0], _ptr(out))
    return out


def rmsnorm_smooth_quant_static(x, fold, scale2, eps=1e-6, apply_norm=True):
    """(RMSNorm with folded weight, or x*fold) then INT8 with the one static scale (clipping past the
    calibrated maximum). Returns (xq, x_scale) with x_scale[t] = delta for every token."""
    x = _need(x, np.uint16, "x")
    T, K = x.shape
    f = _need(fold, np.float32, "fold")
    s2 = _need(scale2, np.float32, "scale2")
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    lib().orc_rmsnorm_smooth_quant_static(_ptr(x), T, K, _ptr(f), float(eps), int(bool(apply_norm)), _ptr(s2),
                                          _ptr(xq), _ptr(xs))
    return xq, xs


def fold_into_prev_linear(w_prev, b_prev, fold):
    """Previous bf16 linear [K, Kp] with its output channel j multiplied by fold[j] ([MIGRATE]
    section 7). Returns (w_out, b_out) as bf16 bits (b_out None without a bias)."""
    w = _need(w_prev, np.uint16, "w_prev")
    K, Kp = w.shape
    f = _need(fold, np.float32, "fold")
    b = None if b_prev is None else _need(b_prev, np.uint16, "b_prev")
    wo = np.empty((K, Kp), np.uint16)
    bo = None if b is None else np.empty(K, np.uint16)
    lib().orc_fold_into_prev_linear(_ptr(w), _ptr(b), K, Kp, _ptr(f), _ptr(wo), _ptr(bo))
    return wo, bo


def fold_into_w_scale(w_scale, fold):
    """Per-output-channel dequantisation scale of an INT8 previous layer times fold (binary32)."""
    ws = _need(w_scale, np.float32, "w_scale")
    f = _need(fold, np.float32, "fold")
    out = np.empty_like(ws)
    lib().orc_fold_into_w_scale(_ptr(ws), ws.shape[0], _ptr(f), _ptr(out))
    return out


def e4m3_encode(a):
    """binary32 -> E4M3 codes (nearest, ties to even, saturating at 448), element by element."""
    a = np.asarray(a, np.float32)
    f = lib().orc_e4m3_encode
    return np.array([f(float(v)) for v in a.ravel()], np.uint8).reshape(a.shape)


def e4m3_decode(c):
    """E4M3 codes -> binary32 values."""
    c = np.asarray(c, np.uint8)
    f = lib().orc_e4m3_decode
    return np.array([f(int(v)) for v in c.ravel()], np.float32).reshape(c.shape)


def smooth_quantize_weight_f8(w, s=None):
    """diag(s)*W then E4M3 per output row (scale max/448). Returns (wq uint8 codes, w_scale)."""
    w = _need(w, np.uint16, "w")
    N, K = w.shape
    wq = np.empty((N, K), np.uint8)
    ws = np.empty(N, np.float32)
    work = np.empty(K, np.float32)
    sv = None if s is None else _need(s, np.float32, "s")
    lib().orc_smooth_quantize_weight_f8(_ptr(w), N, K, _ptr(sv), _ptr(wq), _ptr(ws), _ptr(work))
    return wq, ws


def rmsnorm_smooth_quant_f8(x, fold, eps=1e-6, apply_norm=True):
    """(RMSNorm with folded weight, or x*fold) then E4M3 per token. Returns (xq uint8 codes, x_scale)."""
    x = _need(x, np.uint16, "x")
    T, K = x.shape
    f = _need(fold, np.float32, "fold")
    xq = np.empty((T, K), np.uint8)
    xs = np.empty(T, np.float32)
    work = np.empty(K, np.float32)
    lib().orc_rmsnorm_smooth_quant_f8(_ptr(x), T, K, _ptr(f), float(eps), int(bool(apply_norm)), _ptr(xq), _ptr(xs),
                                      _ptr(work))
    return xq, xs


def gemm_f8(xq, wq, rows=None, cols=None):
    """Exact (binary64) sum of E4M3 products for the listed rows / columns."""
    xq = _need(xq, np.uint8, "xq")
    wq = _need(wq, np.uint8, "wq")
    T, K = xq.shape
    N = wq.shape[0]
    ri = None if rows is None else np.ascontiguousarray(rows, np.int64)
    ci = None if cols is None else np.ascontiguousarray(cols, np.int64)
    nr = T if ri is None else ri.shape[0]
    nc = N if ci is None else ci.shape[0]
    acc = np.empty((nr, nc), np.float64)
    lib().orc_gemm_f8(_ptr(xq), T, _ptr(wq), N, K, _ptr(ri), nr, _ptr(ci), nc, _ptr(acc))
    return acc


def dequant_f32(acc, x_scale, w_scale, bias=None, rows=None, cols=None):
    """bf16(acc * (x_scale[t] * w_scale[n]) + bias[n]) from binary32 accumulators (bf16 bits)."""
    acc = _need(acc, np.float32, "acc")
    xs = _need(x_scale, np.float32, "x_scale")
    ws = _need(w_scale, np.float32, "w_scale")
    b = None if bias is None else _need(bias, np.uint16, "bias")
    ri = None if rows is None else np.ascontiguousarray(rows, np.int64)
    ci = None if cols is None else np.ascontiguousarray(cols, np.int64)
    nr, nc = acc.shape
    y = np.empty((nr, nc), np.uint16)
    lib().orc_dequant_f32(_ptr(acc), _ptr(xs), _ptr(ws), _ptr(b), _ptr(ri), nr, _ptr(ci), nc, _ptr(y))
    return y


def w8a8_linear_f8(xq, x_scale, wq, w_scale, bias=None, rows=None, cols=None):
    """FP8 GEMM (exact accumulation) then the dequant epilogue on the accumulator rounded to binary32.
    Returns (y bf16 bits, acc binary64)."""
    acc = gemm_f8(xq, wq, rows, cols)
    return dequant_f32(acc.astype(np.float32), x_scale, w_scale, bias, rows, cols), acc


def calibrate_absmax_layernorm(a, gamma, beta, eps=1e-5, amax=None, accumulate=False):
    """Per-column abs-max of LayerNorm(a) * gamma + beta ([WOVS] "Integration with Transformers"). Returns amax (float32 [cols])."""
    a = _need(a, np.uint16, "a")
    rows, cols = a.shape
    if amax is None:
        amax = np.zeros(cols, np.float32)
    g = _need(np.asarray(gamma), np.float32, "gamma")
    b = _need(np.asarray(beta), np.float32, "beta")
    work = np.empty(cols, np.float32)
    lib().orc_calibrate_absmax_layernorm(_ptr(a), rows, cols, cols, _ptr(g), _ptr(b), float(eps), _ptr(amax),
                                         int(bool(accumulate)), _ptr(work))
    return amax


def fold_layernorm_bias(beta, s):
    """beta / s (binary32): the LayerNorm bias with S^-1 folded in ([WOVS] "Integration with Transformers")."""
    b = _need(np.asarray(beta), np.float32, "beta")
    sv = _need(np.asarray(s), np.float32, "s")
    out = np.empty_like(b)
    lib().orc_fold_layernorm_bias(_ptr(b), _ptr(sv), b.shape[0], _ptr(out))
    return out


def layernorm_smooth_quant(x, fold, beta_fold, eps=1e-5):
    """LayerNorm with the folded scale and bias, then per-token INT8. Returns (xq, x_scale)."""
    x = _need(x, np.uint16, "x")
    T, K = x.shape
    f = _need(fold, np.float32, "fold")
    bf = _need(beta_fold, np.float32, "beta_fold")
    xq = np.empty((T, K), np.int8)
    xs = np.empty(T, np.float32)
    work = np.empty(2 * K, np.float32)
    lib().orc_layernorm_smooth_quant(_ptr(x), T, K, _ptr(f), _ptr(bf), float(eps), _ptr(xq), _ptr(xs), _ptr(work))
    return xq, xs


def gemm_s8(xq, wq, rows=None, cols=None):
    """acc[t, n] = sum_k xq[t, k] * wq[n, k] (int32) for the listed rows / columns."""
    xq = _need(xq, np.int8, "xq")
    wq = _need(wq, np.int8, "wq")
    T, K = xq.shape
    N = wq.shape[0]
    ri = None if rows is None else np.ascontiguousarray(rows, np.int64)
    ci = None if cols is None else np.ascontiguousarray(cols, np.int64)
    nr = T if ri is None else ri.shape[0]
    nc = N if ci is None else ci.shape[0]
    acc = np.empty((nr, nc), np.int32)
    lib().orc_gemm_s8(_ptr(xq), T, _ptr(wq), N, K, _ptr(ri), nr, _ptr(ci), nc, _ptr(acc))
    return acc


def dequant(acc, x_scale, w_scale, bias=None, rows=None, cols=None):
    """bf16(float(acc) * (x_scale[t] * w_scale[n]) + bias[n]) as uint16 bit patterns."""
    acc = _need(acc, np.int32, "acc")
    xs = _need(x_scale, np.float32, "x_scale")
    ws = _need(w_scale, np.float32, "w_scale")
    b = None if bias is None else _need(bias, np.uint16, "bias")
    ri = None if rows is None else np.ascontiguousarray(rows, np.int64)
    ci = None if cols is None else np.ascontiguousarray(cols, np.int64)
    nr, nc = acc.shape
    y = np.empty((nr, nc), np.uint16)
    lib().orc_dequant(_ptr(acc), _ptr(xs), _ptr(ws), _ptr(b), _ptr(ri), nr, _ptr(ci), nc, _ptr(y))
    return y


def w8a8_linear(xq, x_scale, wq, w_scale, bias=None, rows=None, cols=None):
    """INT8 GEMM then the dequant epilogue. Returns (y bf16 bits, acc int32)."""
    acc = gemm_s8(xq, wq, rows, cols)
    return dequant(acc, x_scale, w_scale, bias, rows, cols), acc


def f32_to_bf16(a):
    """binary32 -> bf16 bits (round to nearest even), element by element through the oracle."""
    a = np.asarray(a, np.float32)
    f = lib().orc_f32_to_bf16
    return np.array([f(float(v)) for v in a.ravel()], np.uint16).reshape(a.shape)


def bf16_to_f32(h):
    """bf16 bits -> binary32 (exact)."""
    h = np.asarray(h, np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)
