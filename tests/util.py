"""Helpers shared by the GPU parity tests: moving seeded inputs to the
device, bit views of bf16, and bf16 ulp distances.  No arithmetic of the
method lives here."""
from __future__ import annotations

import numpy as np
import torch


def bf16_bits_to_torch(bits: np.ndarray, device=None) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device) if device is not None else t


def torch_bf16_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_order(bits: np.ndarray) -> np.ndarray:
    """Map bf16 bit patterns to integers whose difference counts ulps (+0 == -0)."""
    b = bits.astype(np.int32)
    return np.where(b >= 0x8000, -(b & 0x7FFF), b)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(bf16_order(a_bits) - bf16_order(b_bits))


def is_nan_bits(bits: np.ndarray) -> np.ndarray:
    return ((bits & 0x7F80) == 0x7F80) & ((bits & 0x007F) != 0)


def sample_rows(M: int, n: int, seed: int) -> np.ndarray:
    """First, last, tile-boundary and random rows of an M-row problem."""
    fixed = [0, 1, 2, 31, 32, 127, 128, 129, M // 2, M - 129, M - 128, M - 2, M - 1]
    rng = np.random.default_rng(seed)
    extra = rng.choice(M, size=min(n, M), replace=False)
    rows = np.unique(np.array([r for r in fixed if 0 <= r < M] + list(extra), dtype=np.int64))
    return rows


def row_chunks(M: int, chunk: int = 2048):
    """Row slices covering 0..M in pieces of `chunk` rows: full-size oracle
    comparisons run piece by piece, so the oracle's int64 accumulators stay a
    few hundred MB whatever M * N is."""
    return [slice(r, min(M, r + chunk)) for r in range(0, M, chunk)]
