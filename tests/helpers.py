"""Shared helpers of the GPU parity tests: tolerance checks, sampling, sentinels."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

# |gpu - ref| <= RTOL*|ref| + ATOL elementwise, ref in fp64 (bf16 out, fp32 accumulation).
RTOL = 1e-2
ATOL = 1e-2
SENTINEL_I16 = workloads.BF16_SENTINEL - (1 << 16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact fp64 copy of a bf16 tensor (any device)."""
    return oracle.bf16_to_f64(oracle.as_u16(t))


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str):
    """Elementwise tolerance check; NaN or Inf in a checked element fails."""
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    assert np.all(np.isfinite(ref)), f"{what}: oracle value not finite"
    fin = np.isfinite(gpu)
    assert fin.all(), f"{what}: {np.count_nonzero(~fin)} non-finite GPU values"
    err = np.abs(gpu - ref)
    bound = RTOL * np.abs(ref) + ATOL
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {np.count_nonzero(bad)} of {err.size} elements out of "
                             f"tolerance; worst at {i}: gpu={gpu[i]} ref={ref[i]}")


def sentinel(shape, device="cuda") -> torch.Tensor:
    return workloads.sentinel_like(shape, device=device)


def is_sentinel(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16) == SENTINEL_I16


def sample_rows(offs, rows_alloc: int, seed: int, per_group: int = 60) -> np.ndarray:
    """Rows {s, s+1, t-2, t-1} of every non-empty group plus seeded random rows."""
    rng = np.random.default_rng(seed)
    starts, ends, _ = oracle.group_bounds(offs, rows_alloc)
    rows = []
    for s, t in zip(starts, ends):
        if t <= s:
            continue
        rows += [s, min(s + 1, t - 1), max(t - 2, s), t - 1]
        rows += list(rng.integers(s, t, per_group))
    return np.unique(np.asarray(rows, dtype=np.int64))


def sample_k(K: int, seed: int, n: int = 32) -> np.ndarray:
    rng = np.random.default_rng(seed)
    ks = set([0, K - 1]) | set(rng.integers(0, K, n - 2).tolist())
    return np.array(sorted(ks), dtype=np.int64)
