"""Helpers shared by the GPU parity tests: moving bf16 bit patterns between
numpy and torch, the bf16-ulp tolerance, and sampled-row selection."""
from __future__ import annotations

import numpy as np
import torch


def to_dev(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    """CUDA/CPU bf16 tensor -> uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits)."""
    a = np.abs(v.astype(np.float64))
    a = np.where(a < 2.0 ** -126, 2.0 ** -126, a)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check_y(y_bits: np.ndarray, ref_y_bits: np.ndarray, ref_y32: np.ndarray, what: str):
    """The output bar: every y within 1 bf16 ulp of the oracle's fp32 epilogue
    value, all finite.  Returns the number of outputs that are not bit-equal
    to the oracle's bf16 (expected 0)."""
    y = bf16_to_f64(y_bits)
    assert np.isfinite(y).all(), f"{what}: non-finite output"
    err = np.abs(y - ref_y32.astype(np.float64))
    tol = bf16_ulp(ref_y32)
    bad = err > tol
    assert not bad.any(), f"{what}: {int(bad.sum())} outputs beyond 1 bf16 ulp, max err {err.max()}"
    return int((y_bits != ref_y_bits).sum())


def sample_rows(M: int, seed: int = 0, n_random: int = 64, tile: int = 128) -> np.ndarray:
    """Seeded random rows plus the rows on both sides of every tile boundary
    and the last row."""
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n_random, M), replace=False).tolist())
    for b in range(0, M, tile):
        rows.add(b)
        if b > 0:
            rows.add(b - 1)
    rows.add(M - 1)
    return np.array(sorted(rows), dtype=np.int64)
