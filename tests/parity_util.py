"""Shared helpers for the GPU parity tests: move the same seeded arrays to the
device and to the oracle, and compare with the stated tolerances.

Tolerances (fixed for every parity test):
  fp32 inputs:  max |GPU - oracle| <= 1e-5 on Y, dQ, dK, dV, dSink
  bf16 inputs:  Y max abs <= 1e-2; dQ/dK/dV/dKV relative Frobenius <= 2e-2,
                the oracle evaluated on the bf16-rounded inputs in float64.
"""
from __future__ import annotations

import numpy as np
import torch

FP32_ABS = 1e-5
BF16_O_ABS = 1e-2
BF16_GRAD_REL = 2e-2


def to_dev(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to("cuda").to(dtype)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def check_close(name: str, got: np.ndarray, want: np.ndarray, *, fp32: bool, grad: bool,
                row_scale: bool = False):
    if fp32:
        err = float(np.abs(got - want).max()) if got.size else 0.0
        assert err <= FP32_ABS, f"{name}: max abs {err:.3e} > {FP32_ABS}"
    elif grad:
        err = rel_fro(got, want)
        assert err <= BF16_GRAD_REL, f"{name}: rel Frobenius {err:.3e} > {BF16_GRAD_REL}"
    else:
        diff = np.abs(got - want)
        if row_scale and got.size:
            # Rows with a handful of allowed keys have |O| up to the largest
            # |V| entry (about 3-4 for unit normals at d = 128); the bf16
            # rounding of O (half an ulp, 2^-9 relative) and of the P operand
            # both scale with it.
            diff = diff / np.maximum(1.0, np.abs(want).max(axis=-1, keepdims=True))
        err = float(diff.max()) if got.size else 0.0
        assert err <= BF16_O_ABS, f"{name}: max abs {err:.3e} > {BF16_O_ABS}"
    return err
