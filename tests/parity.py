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


def oracle_parallel(fn, N, *args, rows_per_job=256, threads=None):
    """Run an oracle function over row windows on host threads (the C oracle
    releases the GIL); returns the per-window results concatenated along N."""
    import concurrent.futures as cf
    import os
    M = args[-1].shape[0]
    jobs = [(n0, min(N, n0 + rows_per_job)) for n0 in range(0, N, rows_per_job)]
    with cf.ThreadPoolExecutor(max_workers=threads or os.cpu_count() or 1) as ex:
        parts = list(ex.map(lambda j: fn(*args[:-1], args[-1], N, window=(0, M, j[0], j[1])), jobs))
    return parts


def swiglu_tolerance(r, tol=TOL_FP32):
    """Propagated bound for out = silu(g) u: tol (1.1 |u| S_g + |silu(g)| S_u) + 8 ulp(out)."""
    g, u = r["g"], r["u"]
    e = np.exp(-np.abs(g))  # never overflows: silu(g) = g * sigmoid(g), sigmoid from exp(-|g|)
    silu = g * np.where(g >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    ulp = np.spacing(np.abs(r["out"]).astype(np.float32)).astype(np.float64)
    return tol * (1.1 * np.abs(u) * r["Sg"] + np.abs(silu) * r["Su"]) + 8 * ulp
