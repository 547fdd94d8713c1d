"""Seeded synthetic inputs for the ragged MoE grouped GEMM.

This module draws random numbers and lays them out; it holds none of the grouped GEMM's
arithmetic. Both sides of every parity check (the CPU oracle and the CUDA library) take
their inputs from here, so neither side generates inputs for the other.

Shapes and group-size recipes follow the workloads the pages describe:

* ``tiny``: the PyTorch issue 152668 repro ("Easy repro scenario"): E=4, x[48,8], w[4,8,16],
  cumulative end offsets (8,16,32,40) and the empty-expert variant (8,8,32,40); rows 40..47
  lie beyond the last offset.
* ``masked``: the sglang PR 32385 masked down-GEMM ("Evidence", minimal reproduction):
  g=8, mmax=128, k=768, n=2048, per-expert masked_m.
* ``gateup`` / ``downproj``: MoE projections with E=64, N=1536 (sglang PR 32385,
  "Evidence" operand table) and E=32, N=7168.
* ``large`` / ``large_unaligned``: the TileOPs issue 1566 shape ("Summary"): numel=262144,
  N=4096, K=6144.

Values: activations and upstream gradients N(0,1); weights N(0,1/K) (N(0,1) for ``tiny``),
drawn in float32 from a seeded ``torch.Generator`` and rounded to bf16 (round to nearest
even). Group sizes come from ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

BF16_SENTINEL = 0xDEAD  # bit pattern pre-filled into output buffers; -1.955e+18 as bf16

TINY_OFFSETS = (8, 16, 32, 40)        # PyTorch issue 152668 repro: runs
TINY_OFFSETS_EMPTY = (8, 8, 32, 40)   # same repro: expert 1 has no rows

CONFIGS = {
    "tiny": dict(E=4, K=8, N=16, T=40, seed=1),
    "masked": dict(E=8, K=768, N=2048, mmax=128, seed=2),
    "gateup": dict(E=64, K=2048, N=1536, T=32768, seed=3),
    "downproj": dict(E=32, K=2048, N=7168, T=65536, seed=4),
    "large": dict(E=16, K=6144, N=4096, T=262144, seed=5),
    "large_unaligned": dict(E=16, K=6144, N=4096, T=262144, seed=5),
    # two experts of the large shape (1.2 GB on the device): the profiling case of the
    # large-shape kernels
    "large_e2": dict(E=2, K=6144, N=4096, T=32768, seed=6),
}


def offsets_from_sizes(sizes) -> np.ndarray:
    """Cumulative end offsets (int32, length E, no leading zero) for group sizes."""
    s = np.asarray(sizes, dtype=np.int64)
    return np.cumsum(s).astype(np.int32)


def group_sizes(name: str, seed: Optional[int] = None) -> np.ndarray:
    """Seeded group sizes (int64[E]) of a named ragged workload."""
    cfg = CONFIGS[name]
    seed = cfg["seed"] if seed is None else seed
    E, T = cfg["E"], cfg.get("T")
    rng = np.random.default_rng(seed)
    if name == "tiny":
        return np.diff(np.concatenate([[0], np.asarray(TINY_OFFSETS)])).astype(np.int64)
    if name == "gateup":
        # 4 experts forced empty; the other 60 follow Zipf(1.2) weights r^-1.2 over a random
        # rank order; multinomial over T rows; at least one size not a multiple of 8.
        while True:
            zero = rng.choice(E, 4, replace=False)
            live = np.setdiff1d(np.arange(E), zero)
            ranks = rng.permutation(len(live)) + 1
            p = ranks.astype(np.float64) ** -1.2
            p /= p.sum()
            s = rng.multinomial(T, p)
            sizes = np.zeros(E, dtype=np.int64)
            sizes[live] = s
            if np.any(sizes % 8 != 0):
                return sizes
    if name == "downproj":
        # 2 experts forced empty; the other 30 uniform multinomial, redrawn until every live
        # size is > 0 and not a multiple of 128.
        zero = rng.choice(E, 2, replace=False)
        live = np.setdiff1d(np.arange(E), zero)
        while True:
            s = rng.multinomial(T, np.full(len(live), 1.0 / len(live)))
            if np.all(s > 0) and np.all(s % 128 != 0):
                sizes = np.zeros(E, dtype=np.int64)
                sizes[live] = s
                return sizes
    if name in ("large", "large_e2"):
        return np.full(E, T // E, dtype=np.int64)
    if name == "large_unaligned":
        d = rng.integers(1, 128, E // 2)
        base = T // E
        return np.concatenate([base + d, base - d]).astype(np.int64)
    raise KeyError(name)


def masked_counts(seed: int = 2, E: int = 8, mmax: int = 128) -> np.ndarray:
    """masked_m for the masked workload: 8*U{0..16}, one expert at 0 and one at 8."""
    rng = np.random.default_rng(seed)
    m = 8 * rng.integers(0, mmax // 8 + 1, E)
    two = rng.choice(E, 2, replace=False)
    m[two[0]] = 0
    m[two[1]] = 8
    return m.astype(np.int32)


def _randn_bf16(shape, gen: torch.Generator, device, std: float = 1.0,
                chunk_rows: int = 8192) -> torch.Tensor:
    """N(0, std^2) drawn in float32 in row chunks from one generator, rounded to bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    if out.numel() == 0:
        return out
    flat = out.view(shape[0], -1) if len(shape) > 1 else out.view(-1, 1)
    rows = flat.shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0, flat.shape[1]), generator=gen, device=device,
                        dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        flat[r0:r1].copy_(x)
        del x
    return out


def sentinel_like(shape, device="cpu") -> torch.Tensor:
    """A bf16 buffer whose every element has the sentinel bit pattern."""
    t = torch.empty(shape, dtype=torch.int16, device=device)
    t.fill_(BF16_SENTINEL - (1 << 16))
    return t.view(torch.bfloat16)


@dataclasses.dataclass
class RaggedInputs:
    name: str
    E: int
    K: int
    N: int
    sizes: np.ndarray        # int64[E]
    offs: np.ndarray         # int32[E], cumulative ends
    rows_alloc: int
    A: torch.Tensor          # bf16 [rows_alloc, K]
    W: torch.Tensor          # bf16 [E, K, N]
    dY: Optional[torch.Tensor]  # bf16 [rows_alloc, N]

    @property
    def T(self) -> int:
        return int(self.offs[-1]) if len(self.offs) else 0

    @property
    def flops(self) -> int:
        return 2 * int(self.sizes.sum()) * self.K * self.N


@dataclasses.dataclass
class MaskedInputs:
    E: int
    mmax: int
    K: int
    N: int
    masked_m: np.ndarray     # int32[E]
    A: torch.Tensor          # bf16 [E, mmax, K]
    W: torch.Tensor          # bf16 [E, K, N]

    @property
    def flops(self) -> int:
        m = np.clip(self.masked_m.astype(np.int64), 0, self.mmax)
        return 2 * int(m.sum()) * self.K * self.N


def make_ragged_custom(E: int, K: int, N: int, sizes, *, seed: int, tail: int = 0,
                       nan_tail: bool = True, w_std: Optional[float] = None,
                       device="cpu", with_dy: bool = True, name: str = "custom",
                       offs=None) -> RaggedInputs:
    """Ragged inputs for arbitrary sizes. ``tail`` extra rows follow the last group (NaN
    when ``nan_tail``). ``offs`` overrides the offsets (for invalid-offset cases)."""
    sizes = np.asarray(sizes, dtype=np.int64)
    o = offsets_from_sizes(sizes) if offs is None else np.asarray(offs, dtype=np.int32)
    T = int(sizes.sum())
    rows_alloc = T + tail
    gen = torch.Generator(device=device).manual_seed(seed)
    w_std = (1.0 / math.sqrt(K)) if w_std is None else w_std
    A = _randn_bf16((rows_alloc, K), gen, device)
    W = _randn_bf16((E, K, N), gen, device, std=w_std)
    dY = _randn_bf16((rows_alloc, N), gen, device) if with_dy else None
    if nan_tail and tail > 0:
        A[T:] = float("nan")
        if dY is not None:
            dY[T:] = float("nan")
    return RaggedInputs(name, E, K, N, sizes, o, rows_alloc, A, W, dY)


def make_ragged(name: str, *, tail: int = 128, nan_tail: bool = True, device="cpu",
                with_dy: bool = True, seed: Optional[int] = None) -> RaggedInputs:
    """A named ragged workload. Parity runs use a NaN tail of ``tail`` rows past the last
    offset; timing runs pass ``tail=0``."""
    cfg = CONFIGS[name]
    seed = cfg["seed"] if seed is None else seed
    sizes = group_sizes(name, seed)
    w_std = 1.0 if name == "tiny" else None
    if name == "tiny":
        tail = 8  # the repro's x has 48 rows for offsets ending at 40
    return make_ragged_custom(cfg["E"], cfg["K"], cfg["N"], sizes, seed=seed, tail=tail,
                              nan_tail=nan_tail, w_std=w_std, device=device,
                              with_dy=with_dy, name=name)


def make_tiny(offsets=TINY_OFFSETS, *, nan_tail: bool = True, seed: int = 1,
              device="cpu") -> RaggedInputs:
    """The 4-expert M=48/K=8/N=16 repro inputs with the given cumulative end offsets.

    x[48,8], w[4,8,16] and dY[48,16] are N(0,1) and do not depend on the offsets, so every
    offset variant sees the same values. With ``nan_tail`` the rows at and past the last
    offset (clamped to 0..48) are NaN."""
    offs = np.asarray(offsets, dtype=np.int32)
    gen = torch.Generator(device=device).manual_seed(seed)
    A = _randn_bf16((48, 8), gen, device)
    W = _randn_bf16((4, 8, 16), gen, device)
    dY = _randn_bf16((48, 16), gen, device)
    T = int(min(max(int(offs.max()) if len(offs) else 0, 0), 48))
    if nan_tail:
        A[T:] = float("nan")
        dY[T:] = float("nan")
    ends = np.clip(offs.astype(np.int64), 0, 48)
    sizes = np.maximum(np.diff(np.concatenate([[0], np.maximum.accumulate(ends)])), 0)
    return RaggedInputs("tiny", 4, 8, 16, sizes, offs, 48, A, W, dY)


def make_masked(*, seed: int = 2, nan_inactive: bool = True, device="cpu",
                masked_m=None, E: int = 8, mmax: int = 128, K: int = 768,
                N: int = 2048) -> MaskedInputs:
    """The masked layout: A[E,mmax,K], W[E,K,N] ~ N(0,1/K); rows >= masked_m[e] NaN."""
    m = masked_counts(seed, E, mmax) if masked_m is None else np.asarray(masked_m, np.int32)
    gen = torch.Generator(device=device).manual_seed(seed)
    A = _randn_bf16((E, mmax, K), gen, device)
    W = _randn_bf16((E, K, N), gen, device, std=1.0 / math.sqrt(K))
    if nan_inactive:
        for e in range(E):
            lo = int(min(max(int(m[e]), 0), mmax))
            A[e, lo:] = float("nan")
    return MaskedInputs(E, mmax, K, N, m, A, W)


def make_routing(T_tok: int, k: int, E: int, K: int, *, seed: int, zipf: float = 1.2,
                 dropped: int = 0, device="cpu"):
    """Top-k routing of T_tok tokens over E experts: each token picks k distinct experts with
    Zipf(zipf) popularity over a seeded random rank order; `dropped` assignments get id -1.
    Returns (topk_ids int32 [T_tok, k], X bf16 [T_tok, K])."""
    rng = np.random.default_rng(seed)
    ranks = rng.permutation(E) + 1
    p = ranks.astype(np.float64) ** -zipf
    p /= p.sum()
    ids = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T_tok)]).astype(np.int32)
    if dropped:
        flat = ids.reshape(-1)
        flat[rng.choice(flat.size, dropped, replace=False)] = -1
    gen = torch.Generator(device=device).manual_seed(seed)
    X = _randn_bf16((T_tok, K), gen, device)
    return ids, X
