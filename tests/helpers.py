"""Shared test helpers: error metrics and device plumbing (no attention math)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

# Tolerances of the parity bar.
TOL_F32_O = 1e-5        # max |dO| absolute, fp32 inputs
TOL_BF16_REL = 2e-2     # max |d| / max |ref| for O, dQ, dK, dV with bf16 inputs
TOL_LSE = 1e-3          # max |dLSE| absolute (natural log units)


def need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    major, minor = torch.cuda.get_device_capability()
    if (major, minor) != (10, 0):
        pytest.skip(f"needs sm_100 (found sm_{major}{minor})")


def f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def rel_err(x, ref) -> float:
    """max|x - ref| / max|ref|; where the exact result is identically zero (for
    example dQ with a single key, dS = P (dP - D) = 0) the absolute error."""
    x, ref = f64(x), f64(ref)
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    return float(np.max(np.abs(x - ref)) / (scale if scale > 1e-6 else 1.0)) if x.size else 0.0


def abs_err(x, ref) -> float:
    x, ref = f64(x), f64(ref)
    return float(np.max(np.abs(x - ref)))
