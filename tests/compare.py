"""Comparison of the GPU outputs (bf16 O, fp32 LSE) with the fp64 oracle, and the tolerance.

Tolerance (fixed by the requirement this library is built to): on O, max |err| <= 1e-2 and
mean |err| <= 1e-3; on LSE, max |err| <= 1e-3. Nothing is rounded before comparing: the bf16/fp32
GPU values are widened and compared with the fp64 oracle directly. The bf16 output format itself
contributes up to half a bf16 ulp (2^-9 relative) to the O error.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


@dataclasses.dataclass
class Report:
    o_max_abs: float
    o_mean_abs: float
    lse_max_abs: float
    o_max_ulps: float
    n: int

    def ok(self) -> bool:
        return self.o_max_abs <= O_MAX_ABS and self.o_mean_abs <= O_MEAN_ABS and self.lse_max_abs <= LSE_MAX_ABS

    def __str__(self) -> str:
        return (f"O max|err| {self.o_max_abs:.3e} mean|err| {self.o_mean_abs:.3e} (max {self.o_max_ulps:.1f} bf16 ulp), "
                f"LSE max|err| {self.lse_max_abs:.3e}, rows {self.n}")


def _bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    return np.exp2(np.floor(np.log2(ax)) - 7)


def compare(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref: np.ndarray, lse_ref: np.ndarray) -> Report:
    """o_gpu: [..., D] bf16 (any device); lse_gpu: [...] fp32; references are fp64 numpy of equal shape."""
    og = o_gpu.detach().to("cpu").to(torch.float64).numpy().reshape(o_ref.shape)
    lg = lse_gpu.detach().to("cpu").to(torch.float64).numpy().reshape(lse_ref.shape)
    if not (np.all(np.isfinite(og)) and np.all(np.isfinite(lg))):
        return Report(float("inf"), float("inf"), float("inf"), float("inf"), int(lse_ref.size))
    err = np.abs(og - o_ref)
    return Report(float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0,
                  float(np.abs(lg - lse_ref).max(initial=0.0)),
                  float((err / _bf16_ulp(o_ref)).max(initial=0.0)), int(lse_ref.size))
