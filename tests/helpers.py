"""Shared helpers for the parity tests: bf16 bit patterns, row sampling, metrics."""
from __future__ import annotations

import math

import numpy as np
import torch

from bit_attention_video_02_b200 import workloads as W


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 numpy copy of a bf16 tensor's bit patterns."""
    return W.bf16_bits(t)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cosine(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / max(np.linalg.norm(a) * np.linalg.norm(b), 1e-300))


def psnr(test, ref) -> float:
    """10 log10(max|ref|^2 / MSE), peak = largest magnitude of the reference."""
    test = np.asarray(test, np.float64)
    ref = np.asarray(ref, np.float64)
    mse = float(np.mean((test - ref) ** 2))
    peak = float(np.max(np.abs(ref)))
    return float("inf") if mse == 0 else 10.0 * math.log10(peak * peak / mse)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def sample_rows(N: int, n: int, seed: int) -> np.ndarray:
    """Seeded query rows, always including the first and last rows (ragged tail)."""
    if n >= N:
        return np.arange(N, dtype=np.int32)
    rng = np.random.default_rng(seed)
    r = rng.choice(N, size=n - 2, replace=False)
    return np.unique(np.concatenate([r, [0, N - 1]])).astype(np.int32)
