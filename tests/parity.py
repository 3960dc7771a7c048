"""Helpers for the GPU parity tests: upload seeded inputs, compare with the oracle.

Tolerances (per output, S = sum_k |w_k x_k| from the oracle):
  fp32-accumulated paths     |gpu - oracle| <= 1e-5 * S     (and exactly 0 where S == 0)
  bf16 tensor-core prefill   |gpu - oracle| <= 4e-3 * S
"""
from __future__ import annotations

import numpy as np
import torch

TOL_FP32 = 1e-5
TOL_BF16 = 4e-3


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def assert_within(got: np.ndarray, ref: np.ndarray, S: np.ndarray, tol: float, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    err = np.abs(got - ref)
    bound = tol * S
    bad = err > bound
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outputs outside tolerance; worst at {i}: "
                             f"gpu={got[i]!r} oracle={ref[i]!r} err={err[i]:.3e} bound={bound[i]:.3e}")
    return float(np.max(err / np.maximum(S, 1e-300)))
