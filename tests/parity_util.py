"""Shared helpers for the GPU parity tests: move the same seeded arrays to the
device and to the oracle, and compare with the stated tolerances.

Tolerances (fixed for every parity test):
  fp32 inputs:  max |GPU - oracle| <= 1e-5 on Y, dQ, dK, dV, dSink
  bf16 inputs:  Y element by element |GPU - oracle| <= 1e-2 + ulp(oracle)/2,
                the ulp of the 16-bit storage type at the reference value
                (the stored Y is the fp32 result rounded to that type, whose
                half ulp exceeds 1e-2 once |Y| >= 4 in bf16); dQ/dK/dV/dKV
                relative Frobenius <= 2e-2, the oracle evaluated on the
                bf16-rounded inputs in float64.
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


def half_ulp(want: np.ndarray, storage: str = "bf16") -> np.ndarray:
    """Half a unit in the last place of the 16-bit storage type ("bf16": 8
    significant bits, smallest normal 2^-126; "f16": 11 bits, smallest normal
    2^-14, below which the spacing stays 2^-24) at each value of `want`."""
    mant, exp = np.frexp(np.abs(np.asarray(want, np.float64)))  # |want| = mant 2^exp, mant in [0.5, 1)
    bits, emin = (8, -126) if storage == "bf16" else (11, -14)
    exp = np.where(mant > 0, np.maximum(exp, emin + 1), emin + 1)  # subnormals and 0: the smallest binade's spacing
    return np.ldexp(1.0, exp - 1 - bits)


def o_excess(got: np.ndarray, want: np.ndarray, storage: str = "bf16", p_abs: np.ndarray | None = None) -> float:
    """Largest |got - want| - ulp(want)/2 over the elements: the part of each
    element's error that the storage rounding of the output cannot explain.
    The bf16 bound is o_excess <= 1e-2.

    p_abs (optional, the oracle's sum_j p~_ij |V_jc| for each element): also
    subtract the largest error the 16-bit rounding of the P operand can make,
    2^-8 p_abs in bf16 (2^-11 in fp16): each P entry is off by at most that
    relative amount while the normaliser l sums the unrounded values. Used
    only where a test forces rows dominated by one key of large |V|, where
    that rounding alone exceeds 1e-2."""
    if not got.size:
        return 0.0
    err = np.abs(got - want) - half_ulp(want, storage)
    if p_abs is not None:
        err = err - p_abs * (2.0 ** -8 if storage == "bf16" else 2.0 ** -11)
    return float(err.max())


def check_close(name: str, got: np.ndarray, want: np.ndarray, *, fp32: bool, grad: bool,
                storage: str = "bf16"):
    if fp32:
        err = float(np.abs(got - want).max()) if got.size else 0.0
        assert err <= FP32_ABS, f"{name}: max abs {err:.3e} > {FP32_ABS}"
    elif grad:
        err = rel_fro(got, want)
        assert err <= BF16_GRAD_REL, f"{name}: rel Frobenius {err:.3e} > {BF16_GRAD_REL}"
    else:
        err = o_excess(got, want, storage)
        assert err <= BF16_O_ABS, f"{name}: |got - want| - ulp(want)/2 = {err:.3e} > {BF16_O_ABS}"
    return err
