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
"""
from __future__ import annotations

from typing import Callable, Iterable, Optional, Sequence

import torch

from . import sq


class SmoothedW8A8Linear:
    """Smoothed W8A8 linear for the weights ``weights`` (bf16 [N_i, K] each, nn.Linear layout).

    gamma:  the RMSNorm weight feeding the group (fp32 [K]), or None for an input used directly
            (then 1/s multiplies the input instead of being folded into a norm).
    bias:   optional bf16 [sum N_i].
    """

    def __init__(self, weights: Sequence[torch.Tensor], alpha: float, gamma: Optional[torch.Tensor] = None,
                 bias: Optional[torch.Tensor] = None, eps: float = 1e-6):
        ws = list(weights)
        self.weight = ws[0] if len(ws) == 1 else torch.cat(ws, dim=0).contiguous()
        self.splits = [w.shape[0] for w in ws]
        self.N, self.K = self.weight.shape
        self.alpha = float(alpha)
        self.gamma = gamma
        self.bias = bias
        self.eps = float(eps)
        dev = self.weight.device
        self.amax_x = torch.zeros(self.K, dtype=torch.float32, device=dev)
        self.amax_w = torch.zeros(self.K, dtype=torch.float32, device=dev)
        self.s = torch.empty(self.K, dtype=torch.float32, device=dev)
        self.fold = torch.empty(self.K, dtype=torch.float32, device=dev)
        self.wq = torch.empty(self.N, self.K, dtype=torch.int8, device=dev)
        self.w_scale = torch.empty(self.N, dtype=torch.float32, device=dev)
        self._seen = 0

    # ------------------------------------------------------------------ offline
    def observe(self, batch: torch.Tensor, stream=None) -> None:
        """Fold one calibration batch (bf16 [rows, K]) into the running activation abs-max."""
        sq.sq_calibrate_absmax(batch, norm_gamma=self.gamma, eps=self.eps, amax=self.amax_x,
                               accumulate=self._seen > 0, stream=stream)
        self._seen += 1

    def finalize(self, reduce_max: Optional[Callable[[torch.Tensor], None]] = None, alpha: Optional[float] = None,
                 smooth: bool = True, stream=None) -> None:
        """Weight abs-max, smoothing factors, fold and the INT8 weight.

        reduce_max: in-place max-reduction of the activation abs-max across data-parallel ranks
                    (each rank observed its own share of the calibration tokens).
        smooth:     False gives the unsmoothed W8A8 baseline (s = 1).
        """
        if reduce_max is not None:
            reduce_max(self.amax_x)
        sq.sq_calibrate_absmax(self.weight, amax=self.amax_w, accumulate=False, stream=stream)
        a = self.alpha if alpha is None else float(alpha)
        sq.sq_compute_scales(self.amax_x, self.amax_w, a, gamma=self.gamma, s=self.s, fold=self.fold, stream=stream)
        if not smooth:
            self.s.fill_(1.0)
            if self.gamma is not None:
                self.fold.copy_(self.gamma)
            else:
                self.fold.fill_(1.0)
        sq.sq_smooth_quantize_weight(self.weight, s=self.s if smooth else None, wq=self.wq, w_scale=self.w_scale,
                                     stream=stream)

    def calibrate(self, batches: Iterable[torch.Tensor], reduce_max=None, stream=None) -> None:
        self._seen = 0
        for b in batches:
            self.observe(b, stream=stream)
        self.finalize(reduce_max=reduce_max, stream=stream)

    # ------------------------------------------------------------------ online
    def quantize_input(self, x: torch.Tensor, xq=None, x_scale=None, stream=None):
        return sq.sq_rmsnorm_smooth_quant(x, self.fold, eps=self.eps, apply_norm=self.gamma is not None,
                                          xq=xq, x_scale=x_scale, stream=stream)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None, xq=None, x_scale=None,
                acc_out=None, stream=None) -> torch.Tensor:
        xq, xs = self.quantize_input(x, xq=xq, x_scale=x_scale, stream=stream)
        return sq.sq_w8a8_linear(xq, xs, self.wq, self.w_scale, bias=self.bias, y=y, acc_out=acc_out, stream=stream)

    __call__ = forward

    def split_output(self, y: torch.Tensor):
        """Views of the fused output per projection (q, k, v or gate, up)."""
        return torch.split(y, self.splits, dim=1)
