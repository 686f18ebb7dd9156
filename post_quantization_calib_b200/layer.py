"""Host-side orchestration of the libsq calls for one smoothing group.

The object mirrors the shape of the layer the pages describe -- offline ``calibrate`` (abs-maxima,
smoothing factors, smoothed INT8 weight) and online ``forward`` (fused RMSNorm + per-token INT8,
W8A8 GEMM with dequant epilogue) -- as in the flowchart of the "System Architecture" section of
"Taming the Outliers: A Deep Dive into SmoothQuant for LLM Quantization". Every arithmetic step is a
libsq kernel; this module only sequences the calls and owns the device buffers.

One smoothing group is the set of projections reading the same normalised input ("SmoothQuant and
W8A8: Quantizing Activations Too", "The trick: move the range into the weights": input_layernorm
feeds q/k/v, post_attention_layernorm feeds gate/up). Their weights share one s, so they are
concatenated along the output dimension and quantised and multiplied as one matrix.

Options beside the RMSNorm-fed, per-token INT8 layer: a LayerNorm in front (S^-1 folded into its gamma
and beta: "SmoothQuant: Weight-Only vs W8A8", "Integration with Transformers"), an input used directly
(1/s multiplies it, or is folded into the previous linear layer with ``fold_into_previous``), one static
per-tensor activation scale, or FP8 E4M3 codes ("SmoothQuant and W8A8...", "One layer, measured").
"""
from __future__ import annotations

from typing import Callable, Iterable, Optional, Sequence

import torch

from . import sq


class SmoothedW8A8Linear:
    """Smoothed W8A8 linear for the weights ``weights`` (bf16 [N_i, K] each, nn.Linear layout).

    gamma:  the weight of the norm feeding the group (fp32 [K]), or None for an input used directly
            (then 1/s multiplies the input instead of being folded into a norm).
    beta:   with norm="layer", the LayerNorm bias (fp32 [K], optional).
    norm:   "rms" (RMSNorm, the default when gamma is given) or "layer" (LayerNorm).
    scheme: "int8" (one dynamic scale per token), "int8_static" (one static per-tensor scale from the
            calibration tokens) or "fp8" (E4M3 codes, one dynamic scale per token).
    bias:   optional bf16 [sum N_i].
    """

    SCHEMES = ("int8", "int8_static", "fp8")

    def __init__(self, weights: Sequence[torch.Tensor], alpha: float, gamma: Optional[torch.Tensor] = None,
                 bias: Optional[torch.Tensor] = None, eps: Optional[float] = None, norm: Optional[str] = None,
                 beta: Optional[torch.Tensor] = None, scheme: str = "int8"):
        if scheme not in self.SCHEMES:
            raise ValueError(f"scheme must be one of {self.SCHEMES}")
        if norm is None:
            norm = "rms" if gamma is not None else "none"
        if norm not in ("rms", "layer", "none"):
            raise ValueError("norm must be 'rms', 'layer' or None")
        if (norm == "none") != (gamma is None):
            raise ValueError("gamma is required with a norm and not used without one")
        if beta is not None and norm != "layer":
            raise ValueError("beta belongs to a LayerNorm (norm='layer')")
        if norm == "layer" and scheme != "int8":
            raise ValueError("the LayerNorm-fed layer is available with scheme 'int8'")
        ws = list(weights)
        self.weight = ws[0] if len(ws) == 1 else torch.cat(ws, dim=0).contiguous()
        self.splits = [w.shape[0] for w in ws]
        self.N, self.K = self.weight.shape
        self.alpha = float(alpha)
        self.gamma = gamma
        self.beta = beta
        self.norm = norm
        self.scheme = scheme
        self.bias = bias
        self.eps = float(eps) if eps is not None else (1e-5 if norm == "layer" else 1e-6)
        dev = self.weight.device
        self.amax_x = torch.zeros(self.K, dtype=torch.float32, device=dev)
        self.amax_w = torch.zeros(self.K, dtype=torch.float32, device=dev)
        self.s = torch.empty(self.K, dtype=torch.float32, device=dev)
        self.fold = torch.empty(self.K, dtype=torch.float32, device=dev)
        self.beta_fold: Optional[torch.Tensor] = None
        self.scale2: Optional[torch.Tensor] = None           # int8_static: {delta, 127/m}
        code_dtype = torch.uint8 if scheme == "fp8" else torch.int8
        self.wq = torch.empty(self.N, self.K, dtype=code_dtype, device=dev)
        self.w_scale = torch.empty(self.N, dtype=torch.float32, device=dev)
        self._seen = 0
        self._input_folded = False

    # ------------------------------------------------------------------ offline
    def _absmax(self, batch, amax, accumulate, stream, fold=None):
        if self.norm == "layer":
            sq.sq_calibrate_absmax_layernorm(batch, self.gamma, self.beta, eps=self.eps, amax=amax,
                                             accumulate=accumulate, stream=stream)
        else:
            g = self.gamma if fold is None else fold
            sq.sq_calibrate_absmax(batch, norm_gamma=g if self.norm == "rms" else None, eps=self.eps, amax=amax,
                                   accumulate=accumulate, stream=stream)

    def observe(self, batch: torch.Tensor, stream=None) -> None:
        """Fold one calibration batch (bf16 [rows, K]) into the running activation abs-max."""
        self._absmax(batch, self.amax_x, self._seen > 0, stream)
        self._seen += 1

    def finalize(self, reduce_max: Optional[Callable[[torch.Tensor], None]] = None, alpha: Optional[float] = None,
                 smooth: bool = True, stream=None, *, _weight_absmax_done: bool = False) -> None:
        """Weight abs-max, smoothing factors, fold and the quantised weight.

        reduce_max: in-place max-reduction of the activation abs-max across data-parallel ranks
                    (each rank observed its own share of the calibration tokens).
        smooth:     False gives the unsmoothed W8A8 baseline (s = 1).
        """
        if reduce_max is not None:
            reduce_max(self.amax_x)
        if not _weight_absmax_done:
            sq.sq_calibrate_absmax(self.weight, amax=self.amax_w, accumulate=False, stream=stream)
        a = self.alpha if alpha is None else float(alpha)
        sq.sq_compute_scales(self.amax_x, self.amax_w, a, gamma=self.gamma, s=self.s, fold=self.fold, stream=stream)
        if not smooth:
            self.s.fill_(1.0)
            if self.gamma is not None:
                self.fold.copy_(self.gamma)
            else:
                self.fold.fill_(1.0)
        s = self.s if smooth else None
        if self.norm == "layer" and self.beta is not None:
            self.beta_fold = sq.sq_fold_layernorm_bias(self.beta, self.s, stream=stream)
        if self.scheme == "fp8":
            sq.sq_smooth_quantize_weight_fp8(self.weight, s=s, wq=self.wq, w_scale=self.w_scale, stream=stream)
        else:
            sq.sq_smooth_quantize_weight(self.weight, s=s, wq=self.wq, w_scale=self.w_scale, stream=stream)

    def calibrate(self, batches: Iterable[torch.Tensor], reduce_max=None, stream=None) -> None:
        """Both offline passes: abs-maxima, then factors and weight; the static scheme reads the
        calibration batches a second time, for the maximum of the activation as it is quantised."""
        batches = list(batches)
        self._seen = 0
        # the first batch and the weight share one launch (both maxima overwritten); LayerNorm-fed
        # inputs take their own calibration kernel
        paired = bool(batches) and self.norm != "layer"
        for i, b in enumerate(batches):
            if i == 0 and paired:
                sq.sq_calibrate_absmax_pair(b, self.weight, norm_gamma=self.gamma if self.norm == "rms" else None,
                                            eps=self.eps, amax=self.amax_x, amax_w=self.amax_w, accumulate=False,
                                            stream=stream)
                self._seen += 1
            else:
                self.observe(b, stream=stream)
        self.finalize(reduce_max=reduce_max, stream=stream, _weight_absmax_done=paired)
        if self.scheme == "int8_static":
            if self.norm == "rms":
                amax_y = torch.empty(self.K, dtype=torch.float32, device=self.weight.device)
                for i, b in enumerate(batches):
                    self._absmax(b, amax_y, i > 0, stream, fold=self.fold)
                if reduce_max is not None:
                    reduce_max(amax_y)
                self.scale2 = sq.sq_static_scale(amax_y, stream=stream)
            else:        # input used directly: max |x * f| = fl(max |x| * |f|), rounding being monotone
                self.scale2 = sq.sq_static_scale(self.amax_x, factor=self.fold, stream=stream)

    def fold_into_previous(self, w_prev: torch.Tensor, b_prev: Optional[torch.Tensor] = None, stream=None):
        """For an input used directly: fold 1/s into the previous linear layer (bf16 [K, Kp] weight and
        optional bias, rewritten in place) and quantise this layer's input with factor 1 from then on."""
        if self.norm != "none":
            raise ValueError("only an input used directly has a previous linear layer to fold into")
        sq.sq_fold_into_prev_linear(w_prev, self.fold, b_prev, w_out=w_prev, b_out=b_prev, stream=stream)
        self.fold.fill_(1.0)
        self._input_folded = True

    # ------------------------------------------------------------------ online
    def quantize_input(self, x: torch.Tensor, xq=None, x_scale=None, stream=None):
        if self.norm == "layer":
            return sq.sq_layernorm_smooth_quant(x, self.fold, self.beta_fold, eps=self.eps, xq=xq, x_scale=x_scale,
                                                stream=stream)
        apply = self.norm == "rms"
        if self.scheme == "fp8":
            return sq.sq_rmsnorm_smooth_quant_fp8(x, self.fold, eps=self.eps, apply_norm=apply, xq=xq, x_scale=x_scale,
                                                  stream=stream)
        if self.scheme == "int8_static":
            if self.scale2 is None:
                raise RuntimeError("calibrate() first: the static scale comes from the calibration tokens")
            return sq.sq_rmsnorm_smooth_quant_static(x, self.fold, self.scale2, eps=self.eps, apply_norm=apply, xq=xq,
                                                     x_scale=x_scale, stream=stream)
        return sq.sq_rmsnorm_smooth_quant(x, self.fold, eps=self.eps, apply_norm=apply, xq=xq, x_scale=x_scale,
                                          stream=stream)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, xq=None, x_scale=None,
                acc_out=None, stream=None) -> torch.Tensor:
        xq, xs = self.quantize_input(x, xq=xq, x_scale=x_scale, stream=stream)
        gemm = sq.sq_w8a8_linear_fp8 if self.scheme == "fp8" else sq.sq_w8a8_linear
        return gemm(xq, xs, self.wq, self.w_scale, bias=self.bias, y=y, acc_out=acc_out, stream=stream)

    __call__ = forward

    def split_output(self, y: torch.Tensor):
        """Views of the fused output per projection (q, k, v or gate, up)."""
        return torch.split(y, self.splits, dim=1)
