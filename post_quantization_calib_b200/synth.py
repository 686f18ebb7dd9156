"""Seeded synthetic inputs for the smoothed W8A8 linear, and the workload table.

This module only draws random tensors; it holds none of the method's arithmetic. Both the CUDA
path and the CPU oracle consume what it returns, so it is the one module they share.

Shape of the data (the pages' description of LLM activations):
  * activations: N(0, 1) tokens in which a fixed, seeded set of input channels is scaled up by
    10-100x -- the same few channels are large in every token ("SmoothQuant and W8A8: Quantizing
    Activations Too", section "Why activations are the hard part"); the generator pattern (randn, a randperm-chosen fraction of channels multiplied
    by a large factor) is the one in the "Implementation in PyTorch" section of "Taming the
    Outliers: A Deep Dive into SmoothQuant for LLM Quantization".
  * weights: N(0, 0.02), roughly normal with no dominant channel ("06 -- SmoothQuant: Migrating
    Difficulty from Activations to Weights", section 1).
  * norm weights gamma = 1 + 0.1 * N(0, 1) for the layers fed by an RMSNorm.
The same outlier channels and factors are used for calibration and for the online tokens.
Large calibration sets are drawn in independently seeded chunks so they can be streamed.
"""
from __future__ import annotations

import dataclasses
from typing import Iterator, List, Optional, Sequence, Tuple

import torch

__all__ = ["OutlierSpec", "Workload", "WORKLOADS", "workload", "outlier_channels",
           "outlier_tokens", "normal_weight", "norm_gamma", "bias_vector", "calibration_chunks",
           "seed_for"]


@dataclasses.dataclass(frozen=True)
class OutlierSpec:
    """Which fraction / how many input channels are outliers and by what factor."""
    count: int                 # number of outlier channels
    lo: float                  # factors drawn U[lo, hi]
    hi: float
    pinned: Optional[float] = None   # if set, the first outlier channel gets exactly this factor


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, calibration size, alpha and data spec."""
    name: str
    index: int
    T: int                      # online tokens
    K: int                      # input channels (hidden size)
    Ns: Tuple[int, ...]         # output width of each smoothing group's fused GEMM
    calib_rows: int             # calibration tokens in total
    calib_chunk: int            # calibration tokens per streamed chunk
    alpha: float
    outliers: OutlierSpec
    norm: bool                  # input comes out of an RMSNorm (1/s folded into its weight)
    bias: bool
    eps: float = 1e-6
    groups: int = 1             # independent smoothing groups (each with its own norm / input)
    decode_T: Tuple[int, ...] = ()

    @property
    def N(self) -> int:
        """Output channels over all smoothing groups."""
        return int(sum(self.Ns))

    def group_N(self, g: int) -> int:
        """Output channels of smoothing group g (one fused GEMM per group)."""
        return int(self.Ns[g])

    def linear_ops(self, T: Optional[int] = None) -> int:
        """2 x multiply-adds of all the workload's GEMMs at T tokens (default: the workload's T)."""
        return 2 * (self.T if T is None else T) * self.N * self.K


def _w(name, index, **kw) -> Workload:
    return Workload(name=name, index=index, **kw)


# The five workloads. Sizes follow the layer shapes the pages discuss (a Qwen3-8B / Llama-style
# 4096-wide block, a 70B-class 8192-wide MLP) and decode-sized token counts.
WORKLOADS: List[Workload] = [
    _w("single_linear_t256_k1024_n1024", 0, T=256, K=1024, Ns=(1024,), calib_rows=8 * 256,
       calib_chunk=256, alpha=0.5, outliers=OutlierSpec(8, 50.0, 50.0), norm=False, bias=True),
    _w("qproj_t8192_k4096_n4096", 1, T=8192, K=4096, Ns=(4096,), calib_rows=128 * 512,
       calib_chunk=8192, alpha=0.5, outliers=OutlierSpec(16, 10.0, 25.0, pinned=25.0),
       norm=True, bias=False),
    _w("block_prefill_t4096_k4096_qkv6144_gateup28672", 2, T=4096, K=4096,
       Ns=(4096 + 1024 + 1024, 2 * 14336), calib_rows=128 * 512, calib_chunk=8192, alpha=0.5,
       outliers=OutlierSpec(41, 10.0, 100.0), norm=True, bias=False, groups=2),
    _w("decode_k4096_n14336", 3, T=64, K=4096, Ns=(14336,), calib_rows=128 * 512,
       calib_chunk=8192, alpha=0.85, outliers=OutlierSpec(16, 10.0, 25.0, pinned=25.0),
       norm=True, bias=False, decode_T=(1, 8, 32, 64)),
    _w("mlp_up_t16384_k8192_n28672", 4, T=16384, K=8192, Ns=(28672,), calib_rows=128 * 2048,
       calib_chunk=8192, alpha=0.5, outliers=OutlierSpec(41, 50.0, 100.0), norm=True, bias=False),
]


def workload(name_or_index) -> Workload:
    if isinstance(name_or_index, int):
        return WORKLOADS[name_or_index]
    for w in WORKLOADS:
        if w.name == name_or_index:
            return w
    raise KeyError(name_or_index)


# Independent random streams per workload.
_STREAMS = {"outliers": 0, "calib": 1, "x": 2, "w": 3, "gamma": 4, "bias": 5}


def seed_for(index: int, stream: str, sub: int = 0, rank: int = 0) -> int:
    """Deterministic seed: workload 1000+index, stream, chunk / group number and rank."""
    return ((1000 + index) * 1_000_003 + _STREAMS[stream] * 10_007 + sub * 101 + rank * 7_919) % (2**62)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def outlier_channels(K: int, spec: OutlierSpec, seed: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Seeded outlier channel indices (randperm) and their factors (CPU tensors)."""
    g = _gen(seed, "cpu")
    idx = torch.randperm(K, generator=g)[: spec.count]
    fac = spec.lo + (spec.hi - spec.lo) * torch.rand(spec.count, generator=g, dtype=torch.float64)
    if spec.pinned is not None and spec.count > 0:
        fac[0] = spec.pinned
    return idx, fac.to(torch.float32)


def outlier_tokens(rows: int, K: int, channels: Tuple[torch.Tensor, torch.Tensor], seed: int,
                   device="cpu") -> torch.Tensor:
    """bf16 [rows, K]: N(0,1) with the outlier channels multiplied by their factors."""
    g = _gen(seed, device)
    x = torch.randn(rows, K, generator=g, device=device, dtype=torch.float32)
    idx, fac = channels
    if idx.numel():
        x[:, idx.to(device)] *= fac.to(device)
    return x.to(torch.bfloat16)


def normal_weight(N: int, K: int, seed: int, device="cpu", std: float = 0.02) -> torch.Tensor:
    """bf16 [N, K] ~ N(0, std^2) (nn.Linear orientation: output channel n, input channel k)."""
    g = _gen(seed, device)
    return (torch.randn(N, K, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def norm_gamma(K: int, seed: int, device="cpu") -> torch.Tensor:
    """float32 [K] RMSNorm weight 1 + 0.1 * N(0, 1)."""
    g = _gen(seed, device)
    return 1.0 + 0.1 * torch.randn(K, generator=g, device=device, dtype=torch.float32)


def bias_vector(N: int, seed: int, device="cpu", std: float = 0.02) -> torch.Tensor:
    """bf16 [N] ~ N(0, std^2)."""
    g = _gen(seed, device)
    return (torch.randn(N, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def calibration_chunks(w: Workload, channels, device="cpu", group: int = 0, rank: int = 0,
                       rows: Optional[int] = None, chunk: Optional[int] = None,
                       ) -> Iterator[torch.Tensor]:
    """Yield the calibration tokens of workload ``w`` in independently seeded chunks."""
    total = w.calib_rows if rows is None else rows
    step = w.calib_chunk if chunk is None else chunk
    i = 0
    done = 0
    while done < total:
        r = min(step, total - done)
        yield outlier_tokens(r, w.K, channels, seed_for(w.index, "calib", group * 100_000 + i, rank), device)
        done += r
        i += 1


def split_rows(total: int, parts: int) -> Sequence[Tuple[int, int]]:
    """Contiguous [start, stop) ranges splitting ``total`` rows into ``parts`` near-equal shares."""
    base, extra = divmod(total, parts)
    out, start = [], 0
    for p in range(parts):
        n = base + (1 if p < extra else 0)
        out.append((start, start + n))
        start += n
    return out


def group_inputs(w: Workload, g: int = 0, device="cpu", T: Optional[int] = None, rank: int = 0) -> dict:
    """All seeded tensors of smoothing group ``g`` of workload ``w``.

    Returns a dict with ``channels`` (outlier indices, factors), ``gamma`` (fp32 [K] or None),
    ``weight`` (bf16 [N_g, K]), ``bias`` (bf16 [N_g] or None) and ``x`` (bf16 [T, K] online tokens;
    each rank draws its own tokens). Calibration tokens come from ``calibration_chunks``.
    """
    K, N = w.K, w.group_N(g)
    ch = outlier_channels(K, w.outliers, seed_for(w.index, "outliers", g))
    return {
        "channels": ch,
        "gamma": norm_gamma(K, seed_for(w.index, "gamma", g), device) if w.norm else None,
        "weight": normal_weight(N, K, seed_for(w.index, "w", g), device),
        "bias": bias_vector(N, seed_for(w.index, "bias", g), device) if w.bias else None,
        "x": outlier_tokens(w.T if T is None else T, K, ch, seed_for(w.index, "x", g, rank), device),
    }
